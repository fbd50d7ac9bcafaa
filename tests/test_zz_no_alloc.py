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


def _filled_cache(wk, B, Hkv, G, n, seed):
    import torch
    cfg = wk.make_config(B, Hkv, Hkv * G, n + 8, bits=2)
    cache = wk.Cache(cfg)
    g = np.random.default_rng(seed)
    k = torch.from_numpy(g.standard_normal((B, n, Hkv, 128)).astype(np.float32)).cuda()
    v = torch.from_numpy(g.standard_normal((B, n, Hkv, 128)).astype(np.float32)).cuda()
    cache.append(k, v)
    return cache


def test_noalloc_matches_decode_two_calls(wk):
    import torch
    lib = wk.load()
    cache = _filled_cache(wk, 4, 4, 4, 2000, 0)
    stream = torch.cuda.current_stream().cuda_stream or None
    g = np.random.default_rng(1)
    for call in range(2):
        q = torch.from_numpy(g.standard_normal((4, 16, 128)).astype(np.float32)).cuda()
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
