"""The allocation-free decode entry point against the regular decode.

wushkv_decode_noalloc serves callers that cannot call cudaMalloc while they
decode (allocator hooks, plug-ins whose host owns all device memory, engines
that forbid allocation after start-up): its split-K scratch is a fixed array
inside the library.  Called through the C ABI twice in a row, it must give
the regular entry point's output within the decode tolerance of the parity
tests.  This file is collected last and builds everything it uses itself.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

DECODE_TOL = 2e-3


@pytest.fixture(scope="module")
def wk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_post_b200 import wushkv
    wushkv.load()
    return wushkv


def _filled_cache(wk, B, Hkv, G, n, seed, quantizer=0):
    import torch
    cfg = wk.make_config(B, Hkv, Hkv * G, n + 8, bits=2, quantizer=quantizer)
    cache = wk.Cache(cfg)
    g = np.random.default_rng(seed)
    k = torch.from_numpy(g.standard_normal((B, n, Hkv, 128)).astype(np.float32)).cuda()
    v = torch.from_numpy(g.standard_normal((B, n, Hkv, 128)).astype(np.float32)).cuda()
    cache.append(k, v)
    return cache


# (batch, KV heads, G, tokens, quantizer): QuEST at G = 4; the affine
# quantizer at G = 8 (larger partials); one long sequence of 2 units spread
# over many CTAs each (the partials-per-unit bound is reached)
CASES = [(4, 4, 4, 2000, 0), (2, 2, 8, 1500, 1), (1, 2, 4, 40000, 0)]


@pytest.mark.parametrize("B,Hkv,G,n,quantizer", CASES)
def test_noalloc_matches_decode_two_calls(wk, B, Hkv, G, n, quantizer):
    """Same plan, same arithmetic, same merge order as wushkv_decode: the
    outputs are bitwise equal (and within the decode tolerance, which the
    parity tests hold wushkv_decode to)."""
    import torch
    lib = wk.load()
    cache = _filled_cache(wk, B, Hkv, G, n, 0, quantizer)
    stream = torch.cuda.current_stream().cuda_stream or None
    g = np.random.default_rng(1)
    for call in range(2):
        q = torch.from_numpy(g.standard_normal((B, Hkv * G, 128)).astype(np.float32)).cuda()
        ref = torch.empty_like(q)
        out = torch.full_like(q, float("nan"))
        assert lib.wushkv_decode(q.data_ptr(), cache.handle, ref.data_ptr(), ctypes.c_float(0.0),
                                 stream) == wk.OK
        assert lib.wushkv_decode_noalloc(q.data_ptr(), cache.handle, out.data_ptr(),
                                         ctypes.c_float(0.0), stream) == wk.OK
        torch.cuda.synchronize()
        r, o = ref.cpu().numpy(), out.cpu().numpy()
        err = np.abs(o - r).max() / np.sqrt(np.mean(r ** 2))
        assert np.isfinite(o).all() and err <= DECODE_TOL, (call, err)
        assert torch.equal(out, ref), call
    assert cache.device_status() == 0


def test_noalloc_rejects_oversize_scratch(wk):
    """2048 units x G 8 need at least one split each: 2048 x 8 x 528 B of
    partials exceed the fixed array, so the call is refused, not run."""
    import torch
    lib = wk.load()
    cache = _filled_cache(wk, 256, 8, 8, 16, 2)
    q = torch.zeros((256, 64, 128), dtype=torch.float32, device="cuda")
    out = torch.zeros_like(q)
    st = lib.wushkv_decode_noalloc(q.data_ptr(), cache.handle, out.data_ptr(), ctypes.c_float(0.0),
                                   None)
    assert st == wk.ECAPACITY
    cache.decode(q, out=out)            # the regular entry point serves it
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
