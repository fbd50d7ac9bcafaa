"""The one-call decode step (append 1 token + query transform + decode,
wushkv_decode_step) against the three separate calls and the oracle (needs a
B200)."""
import numpy as np
import pytest

from bit_kv_cache_post_b200 import inputs as I
from oracle import wushkv_oracle as O
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

DECODE_TOL = 2e-3   # max |out - oracle| / RMS(oracle output)


@pytest.fixture(scope="module")
def wk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_post_b200 import wushkv
    wushkv.load()
    return wushkv


CASES = [(4, 2, O.QUEST_INT), (8, 3, O.QUEST_INT), (1, 4, O.AFFINE_PCTCLIP), (2, 2, O.AFFINE_PCTCLIP)]


def _inputs(G, Hkv, B, n0, steps):
    g = np.random.default_rng(7)
    k = g.standard_normal((B, n0 + steps, Hkv, 128)).astype(np.float32)
    k[..., g.choice(128, 8, replace=False)] *= 20.0
    v = g.standard_normal((B, n0 + steps, Hkv, 128)).astype(np.float32)
    q = g.standard_normal((steps, B, Hkv * G, 128)).astype(np.float32)
    T, TinvT = zip(*[I.key_transform(I.WORKLOADS["tiny-gqa4-ctx1024"], 3, h) for h in range(Hkv)])
    return k, v, q, np.stack(T).astype(np.float32), np.stack(TinvT).astype(np.float32)


@pytest.mark.parametrize("G,bits,quantizer", CASES)
def test_step_equals_separate_calls(wk, G, bits, quantizer):
    """bf16 keys through T: steps that cross the sink, fill the window and
    flush (every 8th step) give bit-identical q', outputs and packed caches
    to append + query_transform + decode."""
    import torch
    B, Hkv, n0, steps = 2, 2, 40, 50
    cfg = wk.make_config(B, Hkv, Hkv * G, n0 + steps + 8, bits=bits, quantizer=quantizer,
                         sink=16, recent=24, chunk=8)
    k, v, q, T, TinvT = _inputs(G, Hkv, B, n0, steps)
    kr, vr, qr = H.rounded(k, "bf16"), H.rounded(v, "bf16"), H.rounded(q, "bf16")
    Td, TiTd = torch.from_numpy(T).cuda(), torch.from_numpy(TinvT).cuda()
    a, b = wk.Cache(cfg), wk.Cache(cfg)
    for c in (a, b):
        c.append(H.to_dev(kr[:, :n0], "bf16"), H.to_dev(vr[:, :n0], "bf16"), Td)
    for s in range(steps):
        ks, vs = H.to_dev(kr[:, n0 + s:n0 + s + 1], "bf16"), H.to_dev(vr[:, n0 + s:n0 + s + 1], "bf16")
        qs = H.to_dev(qr[s], "bf16")
        qp_a = torch.empty(qs.shape, dtype=torch.float32, device="cuda")
        out_a = a.decode_step(ks, vs, Td, qs, TiTd, q_prime=qp_a)
        b.append(ks, vs, Td)
        qp_b = wk.query_transform(qs, TiTd)
        out_b = b.decode(qp_b)
        torch.cuda.synchronize()
        assert torch.equal(qp_a, qp_b)
        assert torch.equal(out_a, out_b)
    assert a.tokens() == b.tokens()
    P = a.tokens()[2]
    assert P > 0
    for kv in (0, 1):
        for u in range(B * Hkv):
            for pa, pb in zip(H.unit_packed_planes(a, u, kv, P), H.unit_packed_planes(b, u, kv, P)):
                assert np.array_equal(pa, pb)
            assert np.array_equal(H.unit_meta(a, u, kv, P), H.unit_meta(b, u, kv, P))
    assert a.device_status() == 0 and b.device_status() == 0


@pytest.mark.parametrize("G,bits,quantizer", CASES)
def test_step_matches_oracle(wk, G, bits, quantizer):
    """Keys transformed by the oracle (float64, rounded to fp32) and passed
    without a transform, so both caches are bit-identical: every step's q'
    within 1e-5 relative error and output within the decode tolerance."""
    import torch
    B, Hkv, n0, steps = 2, 2, 40, 50
    cfg = wk.make_config(B, Hkv, Hkv * G, n0 + steps + 8, bits=bits, quantizer=quantizer,
                         sink=16, recent=24, chunk=8)
    k, v, q, T, TinvT = _inputs(G, Hkv, B, n0, steps)
    kt = np.stack([O.transform_keys(H.rounded(k, "bf16")[:, :, h].astype(np.float64), T[h].astype(np.float64))
                   for h in range(Hkv)], axis=2).astype(np.float32)
    vr, qr = H.rounded(v, "bf16"), H.rounded(q, "bf16")
    TiTd = torch.from_numpy(TinvT).cuda()
    a = wk.Cache(cfg)
    oc = O.OracleCache(H.oracle_cfg(cfg))
    a.append(H.to_dev(kt[:, :n0], "f32"), H.to_dev(vr[:, :n0], "f32"), None)
    oc.append(kt[:, :n0], vr[:, :n0], None)
    lib = wk.load()
    worst = 0.0
    for s in range(steps):
        ks, vs = H.to_dev(kt[:, n0 + s:n0 + s + 1], "f32"), H.to_dev(vr[:, n0 + s:n0 + s + 1], "f32")
        qs = H.to_dev(qr[s], "bf16")
        qp = torch.empty(qs.shape, dtype=torch.float32, device="cuda")
        out = torch.empty(qs.shape, dtype=torch.float32, device="cuda")
        st = lib.wushkv_decode_step(a.handle, ks.data_ptr(), vs.data_ptr(), wk.F32, None, qs.data_ptr(),
                                    wk.BF16, TiTd.data_ptr(), qp.data_ptr(), out.data_ptr(), 0.0, None)
        assert st == wk.OK
        oc.append(kt[:, n0 + s:n0 + s + 1], vr[:, n0 + s:n0 + s + 1], None)
        qo = O.query_transform_gqa(qr[s], TinvT.astype(np.float64))
        qg = qp.cpu().numpy()
        assert (np.linalg.norm(qg - qo, axis=-1) / np.linalg.norm(qo, axis=-1)).max() <= 1e-5
        want = oc.decode(qo)
        worst = max(worst, H.rel_rms_err(out.cpu().numpy(), want))
    assert worst <= DECODE_TOL, worst
    assert a.device_status() == 0


def test_step_argument_errors(wk):
    import torch
    cfg = wk.make_config(1, 1, 4, 16, bits=2, sink=4, recent=4, chunk=4)
    c = wk.Cache(cfg)
    k = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    T = torch.eye(128, dtype=torch.float32, device="cuda")[None].contiguous()
    qp = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
    out = torch.empty_like(qp)
    lib = wk.load()
    # misaligned q' -> EINVAL, nothing appended
    st = lib.wushkv_decode_step(c.handle, k.data_ptr(), k.data_ptr(), wk.BF16, T.data_ptr(), q.data_ptr(),
                                wk.BF16, T.data_ptr(), qp.data_ptr() + 4, out.data_ptr(), 0.0, None)
    assert st == wk.EINVAL and c.tokens()[0] == 0
    for _ in range(16):
        c.decode_step(k, k, T, q, T, q_prime=qp, out=out)
    st = lib.wushkv_decode_step(c.handle, k.data_ptr(), k.data_ptr(), wk.BF16, T.data_ptr(), q.data_ptr(),
                                wk.BF16, T.data_ptr(), qp.data_ptr(), out.data_ptr(), 0.0, None)
    assert st == wk.ECAPACITY and c.tokens()[0] == 16
    torch.cuda.synchronize()
    assert c.device_status() == 0
