"""Full-size workloads in the launch configuration bench.py uses, checked
against the oracle on sampled (sequence, KV head) units (needs a B200).

Bar: transformed keys within 1e-3 relative error, key codes mismatching on
at most 1e-4 of elements (rounding-boundary flips), value codes and scales
bit-exact, key scales within one fp16 ulp, decode outputs within 2e-3 of the
output RMS."""
import numpy as np
import pytest

from bit_kv_cache_post_b200 import inputs as I
from oracle import wushkv_oracle as O
from tests import gpu_helpers as H

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


def _oracle_unit(w, bits, quantizer, k_h, v_h, T_h, max_ctx):
    oc = O.OracleCache(O.CacheConfig(1, 1, w.group, max_ctx, bits=bits, quantizer=quantizer,
                                     sink=w.sink, recent=w.recent, chunk=w.chunk,
                                     r_lo=w.r_lo, r_hi=w.r_hi))
    oc.append(k_h[None, :, None], v_h[None, :, None], T_h[None].astype(np.float64))
    return oc


@pytest.fixture(scope="module")
def qwen8b_inputs():
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    n = w.context - 1
    k = I.round_to(np.stack([I.keys(w, 0, b, n) for b in range(w.batch)]), w.dtype)
    v = I.round_to(np.stack([I.values(w, 0, b, n) for b in range(w.batch)]), w.dtype)
    st = [I.step_tokens(w, 0, b, 0) for b in range(w.batch)]
    ks = I.round_to(np.stack([s[0] for s in st]), w.dtype)[:, :, :, :]
    vs = I.round_to(np.stack([s[1] for s in st]), w.dtype)
    qs = I.round_to(np.stack([s[2] for s in st]), w.dtype)
    T, TinvT = I.key_transforms(w, 0)
    return w, k, v, ks, vs, qs, T, TinvT


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_qwen3_8b_layer_decode_step(wk, qwen8b_inputs, bits):
    """The bench step: prefill 8191 tokens, append 1, transform the
    queries, decode -- all 128 units on the GPU; 3 units checked."""
    import torch
    w, k, v, ks, vs, qs, T, TinvT = qwen8b_inputs
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, w.context + 8, bits=bits,
                         sink=w.sink, recent=w.recent, chunk=w.chunk)
    cache = wk.Cache(cfg)
    Td, TinvTd = torch.from_numpy(T).cuda(), torch.from_numpy(TinvT).cuda()
    cache.append(torch.from_numpy(k).cuda().to(torch.bfloat16), torch.from_numpy(v).cuda().to(torch.bfloat16), Td)
    cache.append(torch.from_numpy(ks).cuda().to(torch.bfloat16), torch.from_numpy(vs).cuda().to(torch.bfloat16), Td)
    qp = wk.query_transform(torch.from_numpy(qs).cuda().to(torch.bfloat16), TinvTd)
    out = cache.decode(qp).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    G = w.group
    for b, h in ((0, 0), (7, 3), (15, 7)):
        u = b * w.n_kv_heads + h
        k_h = np.concatenate([k[b, :, h], ks[b, :, h]])
        v_h = np.concatenate([v[b, :, h], vs[b, :, h]])
        oc = _oracle_unit(w, bits, O.QUEST_INT, k_h, v_h, T[h], w.context + 8)
        assert oc.split() == cache.tokens()[1:]
        H.check_unit_transformed(cache, oc, 0, T[h], k_h, u)
        qprime = O.transform_query(qs[b, h * G:(h + 1) * G], TinvT[h].astype(np.float64))
        want = oc.decode(qprime[None])[0]
        assert H.rel_rms_err(out[b, h * G:(h + 1) * G], want) <= DECODE_TOL


def _device_workload(wk, w, bits, quantizer, n_prefill, n_step, samples):
    """Prefill n_prefill device-drawn tokens, append n_step more, decode one
    query; check the sampled units against the oracle."""
    import torch
    k, v = I.device_kv(w, 0, n_prefill)
    ks, vs = I.device_kv(w, 0, n_step, step=0)
    q = I.device_queries(w, 0, 0)
    T, TinvT = I.key_transforms(w, 0)
    max_ctx = n_prefill + n_step
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, max_ctx, bits=bits,
                         quantizer=quantizer, sink=w.sink, recent=w.recent, chunk=w.chunk,
                         clip_lo_rank=w.r_lo, clip_hi_rank=w.r_hi)
    cache = wk.Cache(cfg)
    Td = torch.from_numpy(T).cuda()
    cache.append(k, v, Td)
    cache.append(ks, vs, Td)
    qp = wk.query_transform(q, torch.from_numpy(TinvT).cuda())
    out = cache.decode(qp).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    G = w.group
    for b, h in samples:
        u = b * w.n_kv_heads + h
        k_h = torch.cat([k[b, :, h], ks[b, :, h]]).float().cpu().numpy()
        v_h = torch.cat([v[b, :, h], vs[b, :, h]]).float().cpu().numpy()
        oc = _oracle_unit(w, bits, quantizer, k_h, v_h, T[h], max_ctx)
        assert oc.split() == cache.tokens()[1:]
        H.check_unit_transformed(cache, oc, 0, T[h], k_h, u)
        qh = q[b, h * G:(h + 1) * G].float().cpu().numpy()
        want = oc.decode(O.transform_query(qh, TinvT[h].astype(np.float64))[None])[0]
        assert H.rel_rms_err(out[b, h * G:(h + 1) * G], want) <= DECODE_TOL
    del k, v
    torch.cuda.empty_cache()


def test_qwen3_32b_layer_gqa8(wk):
    """GQA 8, x50 outliers on 4 channels, Laplace values, context 32768."""
    w = I.WORKLOADS["qwen3-32b-layer-b32-ctx32768"]
    _device_workload(wk, w, 2, O.QUEST_INT, w.context - 1, 1, [(0, 0), (31, 5)])


def test_qwen3_4b_long_context_chunk16(wk):
    """One sequence of 131072 tokens, flush chunk 16, a 16-token append."""
    w = I.WORKLOADS["qwen3-4b-b1-ctx131072"]
    _device_workload(wk, w, 2, O.QUEST_INT, w.context - 16, 16, [(0, 2)])


def test_qwen3_8b_stack_layer_affine(wk):
    """One layer of the 36-layer workload: batch 64, prefill 32768, 2-bit
    percentile-clipped affine (ranks 2 and 127), then one decode step."""
    w = I.WORKLOADS["qwen3-8b-stack36-b64-prefill32768"]
    _device_workload(wk, w, 2, O.AFFINE_PCTCLIP, w.context, 1, [(0, 0), (63, 7)])
