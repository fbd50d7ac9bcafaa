"""Bulk bf16 appends with a key transform (the tensor-core append path)
against the CPU oracle (needs a B200).

Sizes are chosen so that every CTA runs several 128-token tiles (both
stages of each ring are reused, so barrier phases wrap), the last tile of
each unit is ragged, and a second bulk append starts inside the recent
window (old ring rows flushed by the FMA kernel, the rest on the tensor
cores)."""
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


def _inputs(seed, B, n, Hkv, laplace=False):
    g = np.random.default_rng(seed)
    k = g.standard_normal((B, n, Hkv, 128)).astype(np.float32)
    for h in range(Hkv):
        k[:, :, h, g.choice(128, 8, replace=False)] *= 20.0
    v = (g.laplace(0.0, 1.0, (B, n, Hkv, 128)) if laplace
         else g.standard_normal((B, n, Hkv, 128))).astype(np.float32)
    q = g.standard_normal((B, 4 * Hkv, 128)).astype(np.float32)
    return H.rounded(k, "bf16"), H.rounded(v, "bf16"), H.rounded(q, "bf16")


def _transforms(Hkv):
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    T, TinvT = I.key_transforms(w, 5)
    return T[:Hkv], TinvT[:Hkv]


def _run(wk, cfg, k, v, q, T, TinvT, schedule, units, decode_on_gpu_state=False):
    import torch
    cache = wk.Cache(cfg)
    Td = torch.from_numpy(T).cuda()
    i = 0
    for step in schedule:
        cache.append(H.to_dev(k[:, i:i + step], "bf16"), H.to_dev(v[:, i:i + step], "bf16"), Td)
        i += step
    qp = wk.query_transform(H.to_dev(q, "bf16"), torch.from_numpy(TinvT).cuda())
    out = cache.decode(qp).cpu().numpy()
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    Hkv, G = cfg.n_kv_heads, cfg.n_q_heads // cfg.n_kv_heads
    mism = []
    for (b, h) in units:
        u = b * Hkv + h
        oc = O.OracleCache(O.CacheConfig(1, 1, G, cfg.max_ctx, bits=cfg.bits,
                                         quantizer=cfg.quantizer, sink=cfg.sink,
                                         recent=cfg.recent, chunk=cfg.chunk,
                                         r_lo=cfg.clip_lo_rank, r_hi=cfg.clip_hi_rank))
        i = 0
        for step in schedule:
            oc.append(k[b:b + 1, i:i + step, h:h + 1], v[b:b + 1, i:i + step, h:h + 1],
                      T[h:h + 1].astype(np.float64))
            i += step
        assert oc.split() == cache.tokens()[1:]
        mism.append(H.check_unit_transformed(cache, oc, 0, T[h], k[b, :, h], u))
        qprime = O.transform_query(q[b, h * G:(h + 1) * G], TinvT[h].astype(np.float64))
        if decode_on_gpu_state:
            # the decode against exact attention over the cache the GPU built
            # (boundary flips of k' codes then cannot enter the comparison)
            Kg, Vg = H.unit_state_from_export(cache, b, h)
            want = O.attention_f64(qprime, Kg, Vg, 1.0 / np.sqrt(128.0))
        else:
            want = oc.decode(qprime[None])[0]
        assert H.rel_rms_err(out[b, h * G:(h + 1) * G], want) <= DECODE_TOL
    return cache, mism


@pytest.mark.parametrize("quantizer", [O.QUEST_INT, O.AFFINE_PCTCLIP])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bulk_prefill(wk, bits, quantizer):
    """One append of 1821 tokens: 1496 packed rows per unit straight from
    the input (11 full tiles and one of 88 rows), 24 tiles per head shared
    by 4 CTAs."""
    B, Hkv, n = 2, 2, 1821
    k, v, q = _inputs(10 * bits + quantizer, B, n, Hkv)
    T, TinvT = _transforms(Hkv)
    cfg = wk.make_config(B, Hkv, 4 * Hkv, n + 16, bits=bits, quantizer=quantizer)
    cache, _ = _run(wk, cfg, k, v, q, T, TinvT, [n], [(b, h) for b in range(B) for h in range(Hkv)])
    assert cache.tokens() == (n, 64, 1496, 261)


@pytest.mark.parametrize("first", [1000, 1001, 1003])
def test_second_bulk_append(wk, first):
    """A bulk append into a cache whose recent window is full: old ring rows
    and the partial first quad go through the FMA kernel, the rest through
    the tensor cores; then a few single-token appends."""
    B, Hkv = 2, 2
    sched = [first, 1900 - first, 1, 1, 5]
    n = sum(sched)
    k, v, q = _inputs(first, B, n, Hkv)
    T, TinvT = _transforms(Hkv)
    cfg = wk.make_config(B, Hkv, 4 * Hkv, n, bits=2, quantizer=O.QUEST_INT)
    _run(wk, cfg, k, v, q, T, TinvT, sched, [(b, h) for b in range(B) for h in range(Hkv)])


def test_many_units_short_prefill(wk):
    """128 units, 3 tiles each (the last of 48 rows), Laplace values, chunk 16,
    affine 2-bit; sampled units."""
    B, Hkv, n = 16, 8, 64 + 256 + 304 + 3
    k, v, q = _inputs(7, B, n, Hkv, laplace=True)
    T, TinvT = _transforms(Hkv)
    cfg = wk.make_config(B, Hkv, 4 * Hkv, n + 32, bits=2, quantizer=O.AFFINE_PCTCLIP, chunk=16)
    cache, _ = _run(wk, cfg, k, v, q, T, TinvT, [n], [(0, 0), (5, 3), (15, 7)])
    assert cache.tokens()[2] == 304


@pytest.mark.parametrize("ranks", [(1, 128), (2, 128), (1, 127)])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bulk_prefill_affine_ranks(wk, bits, ranks):
    """Affine ranks other than (2, 127) that the tensor-core append serves
    (lowest rank <= 2, highest >= 127): the epilogue's branches without the
    second order statistic."""
    B, Hkv, n = 2, 2, 64 + 256 + 8 * 60 + 3
    k, v, q = _inputs(1000 * bits + ranks[0] + ranks[1], B, n, Hkv)
    T, TinvT = _transforms(Hkv)
    cfg = wk.make_config(B, Hkv, 4 * Hkv, n + 16, bits=bits, quantizer=O.AFFINE_PCTCLIP,
                         clip_lo_rank=ranks[0], clip_hi_rank=ranks[1])
    cache, _ = _run(wk, cfg, k, v, q, T, TinvT, [n], [(b, h) for b in range(B) for h in range(Hkv)],
                    decode_on_gpu_state=True)
    H.check_guards(cache)


def test_bulk_prefill_deep_ranks_fma_path(wk):
    """Affine ranks (8, 121) with bf16 keys through T: the FMA append path
    (warp rank selection) against the oracle."""
    B, Hkv, n = 2, 2, 64 + 256 + 8 * 30 + 1
    k, v, q = _inputs(4242, B, n, Hkv)
    T, TinvT = _transforms(Hkv)
    cfg = wk.make_config(B, Hkv, 4 * Hkv, n + 16, bits=2, quantizer=O.AFFINE_PCTCLIP,
                         clip_lo_rank=8, clip_hi_rank=121)
    cache, _ = _run(wk, cfg, k, v, q, T, TinvT, [n - 40] + [1] * 40,
                    [(b, h) for b in range(B) for h in range(Hkv)], decode_on_gpu_state=True)
    H.check_guards(cache)
