"""CUDA path vs the CPU oracle, element by element (needs a B200)."""
import math

import numpy as np
import pytest

from bit_kv_cache_post_b200 import inputs as I
from oracle import wushkv_oracle as O
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# decode tolerance: max |out - oracle| / RMS(oracle output)
DECODE_TOL = 2e-3


@pytest.fixture(scope="module")
def wk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_post_b200 import wushkv
    wushkv.load()
    return wushkv


def _kv(seed, B, n, Hkv, outliers=True):
    g = np.random.default_rng(seed)
    k = g.standard_normal((B, n, Hkv, 128)).astype(np.float32)
    if outliers:
        for h in range(Hkv):
            k[:, :, h, g.choice(128, 8, replace=False)] *= 20.0
    v = g.standard_normal((B, n, Hkv, 128)).astype(np.float32)
    return k, v


SCHEDULE = [1, 5, 64, 3, 1, 1, 200, 7, 1, 1, 1, 1, 300, 13, 102]   # sums to 701


def _append_both(wk, cfg, k, v, T_host, dtype, schedule):
    import torch
    cache = wk.Cache(cfg)
    oc = O.OracleCache(H.oracle_cfg(cfg))
    kr, vr = H.rounded(k, dtype), H.rounded(v, dtype)
    Td = None if T_host is None else torch.from_numpy(T_host).cuda()
    i = 0
    for step in schedule:
        cache.append(H.to_dev(kr[:, i:i + step], dtype), H.to_dev(vr[:, i:i + step], dtype), Td)
        oc.append(kr[:, i:i + step], vr[:, i:i + step], None if T_host is None else T_host.astype(np.float64))
        i += step
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    return cache, oc


@pytest.mark.parametrize("quantizer", [O.QUEST_INT, O.AFFINE_PCTCLIP])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("sched", ["bulk", "steps"])
def test_cache_bitexact_from_oracle_vectors(wk, bits, quantizer, sched):
    """Fed the same fp32 (already transformed) vectors, packed codes, scales
    and fp16 windows are bit-identical, for one bulk append and for a mix of
    single-token and multi-token appends crossing flush boundaries."""
    n = sum(SCHEDULE)
    cfg = wk.make_config(2, 2, 8, 720, bits=bits, quantizer=quantizer)
    k, v = _kv(bits * 10 + quantizer, 2, n, 2)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n] if sched == "bulk" else SCHEDULE)
    H.compare_cache_bitexact(cache, oc)


@pytest.mark.parametrize("chunk", [8, 16])
def test_cache_bitexact_chunk_sizes(wk, chunk):
    n = 64 + 256 + 5 * chunk + 3
    cfg = wk.make_config(1, 3, 3, n + 5, bits=2, chunk=chunk)
    k, v = _kv(7, 1, n, 3)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [1] * 40 + [n - 40])
    H.compare_cache_bitexact(cache, oc)


def test_degenerate_tokens(wk):
    """All-zero tokens (QuEST delta 0 -> codes L/2) and constant tokens
    (affine scale 0 -> codes 0) match the oracle bit for bit."""
    n = 64 + 256 + 16
    for quantizer in (O.QUEST_INT, O.AFFINE_PCTCLIP):
        cfg = wk.make_config(1, 2, 2, n, bits=2, quantizer=quantizer)
        k, v = _kv(3, 1, n, 2)
        k[:, 64:90] = 0.0
        v[:, 64:90, 0] = 1.5
        v[:, 90:100, 1] = -0.0
        cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n])
        H.compare_cache_bitexact(cache, oc)


@pytest.mark.parametrize("ranks", [(1, 128), (8, 121), (3, 124)])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_affine_ranks_bitexact(wk, bits, ranks):
    """Order statistics other than the default (2, 127): the extreme ranks
    (no clipping) and the deepest supported ones, on one bulk append and on
    single-token appends across flushes; then a decode."""
    n = sum(SCHEDULE)
    cfg = wk.make_config(2, 2, 8, 720, bits=bits, quantizer=O.AFFINE_PCTCLIP,
                         clip_lo_rank=ranks[0], clip_hi_rank=ranks[1])
    k, v = _kv(100 * bits + ranks[0], 2, n, 2)
    for sched in ([n], SCHEDULE):
        cache, oc = _append_both(wk, cfg, k, v, None, "f32", sched)
        H.compare_cache_bitexact(cache, oc)
    out, want = _decode_both(wk, cache, oc, 17)
    assert H.rel_rms_err(out, want) <= DECODE_TOL


@pytest.mark.parametrize("quantizer", [O.QUEST_INT, O.AFFINE_PCTCLIP])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_export_matches_oracle(wk, bits, quantizer):
    """wushkv_export unpacks K and V of sink, packed and recent tokens of a
    unit: codes, scales and fp16 rows equal the oracle's state."""
    n = 64 + 256 + 8 * 23 + 5
    cfg = wk.make_config(2, 3, 6, n + 8, bits=bits, quantizer=quantizer)
    k, v = _kv(7 * bits + quantizer, 2, n, 3)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n - 9] + [1] * 9)
    ns, P, nr = oc.split()
    W = cfg.recent + cfg.chunk
    for (b, h) in [(0, 0), (1, 2)]:
        u = b * cfg.n_kv_heads + h
        for kv in (0, 1):
            codes, meta, rows, kinds = cache.export(b, h, kv, 0, n)
            sink = oc.sink_k if kv == 0 else oc.sink_v
            ring = oc.ring_k if kv == 0 else oc.ring_v
            ocodes = oc.codes_k if kv == 0 else oc.codes_v
            ometa = oc.meta_k if kv == 0 else oc.meta_v
            assert np.array_equal(kinds[:ns], np.zeros(ns))
            assert np.array_equal(kinds[ns:ns + P], np.ones(P))
            assert np.array_equal(kinds[ns + P:], np.full(nr, 2))
            assert np.array_equal(rows[:ns], sink[u, :ns].view(np.uint16))
            slots = [(t - cfg.sink) % W for t in range(ns + P, n)]
            assert np.array_equal(rows[ns + P:], ring[u, slots].view(np.uint16))
            assert np.array_equal(codes[ns:ns + P], ocodes[u, :P])
            nm = 2 if quantizer == O.AFFINE_PCTCLIP else 1
            assert np.array_equal(meta[ns:ns + P, :nm], ometa[u, :P, :nm].view(np.uint16))
            assert not codes[:ns].any() and not codes[ns + P:].any() and not rows[ns:ns + P].any()
        # a range starting and ending inside the packed tokens
        codes, _, _, kinds = cache.export(b, h, 0, ns + 5, 70)
        assert np.array_equal(codes, oc.codes_k[u, 5:75]) and np.all(kinds == 1)


def _decode_both(wk, cache, oc, seed, scale=0.0):
    import torch
    cfg = cache.cfg
    q = np.random.default_rng(seed).standard_normal((cfg.batch, cfg.n_q_heads, 128)).astype(np.float32)
    qd = torch.from_numpy(q).cuda()
    out = cache.decode(qd, scale=scale).cpu().numpy()
    want = oc.decode(q.astype(np.float64), None if scale == 0.0 else scale)
    assert cache.device_status() == 0
    H.check_guards(cache)
    return out, want


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("n", [9, 200, 64 + 264, 1200])
def test_decode_matches_oracle(wk, G, n):
    """Decode over a bit-identical cache: sink-only, window-only, first flush
    and a multi-split context, for every supported group size."""
    cfg = wk.make_config(2, 2, 2 * G, n, bits=2)
    k, v = _kv(G * 1000 + n, 2, n, 2)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n])
    out, want = _decode_both(wk, cache, oc, n + G)
    assert H.rel_rms_err(out, want) <= DECODE_TOL


@pytest.mark.parametrize("G", [4, 8])
def test_decode_many_ctas_per_unit(wk, G):
    """Two units of 30000 tokens: every CTA of the grid holds a few items of
    one unit (most warps one item, several none), ~70 partials per unit;
    repeated decodes give the same bits."""
    import torch
    n = 30000
    cfg = wk.make_config(1, 2, 2 * G, n, bits=2)
    k, v = _kv(4000 + G, 1, n, 2)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n])
    out, want = _decode_both(wk, cache, oc, 11)
    assert H.rel_rms_err(out, want) <= DECODE_TOL
    q = torch.from_numpy(np.random.default_rng(11).standard_normal((1, 2 * G, 128)).astype(np.float32)).cuda()
    for _ in range(3):
        assert np.array_equal(cache.decode(q).cpu().numpy(), out)


@pytest.mark.parametrize("quantizer", [O.QUEST_INT, O.AFFINE_PCTCLIP])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_decode_bits_and_quantizers(wk, bits, quantizer):
    n = 64 + 256 + 8 * 70 + 5
    cfg = wk.make_config(2, 2, 8, n, bits=bits, quantizer=quantizer)
    k, v = _kv(bits + 31 * quantizer, 2, n, 2)
    cache, oc = _append_both(wk, cfg, k, v, None, "f32", [n - 3, 1, 1, 1])
    out, want = _decode_both(wk, cache, oc, 5, scale=0.05)
    assert H.rel_rms_err(out, want) <= DECODE_TOL


def test_query_transform_matches_oracle(wk):
    import torch
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    _, TinvT = I.key_transforms(w, 0)
    q = np.random.default_rng(0).standard_normal((3, 32, 128)).astype(np.float32)
    for dtype in ("bf16", "f16", "f32"):
        qr = H.rounded(q, dtype)
        got = wk.query_transform(H.to_dev(qr, dtype), torch.from_numpy(TinvT).cuda()).cpu().numpy()
        want = O.query_transform_gqa(qr, TinvT.astype(np.float64))
        err = np.linalg.norm(got - want, axis=-1) / np.linalg.norm(want, axis=-1)
        assert err.max() <= 1e-5, (dtype, err.max())


def test_end_to_end_with_transform(wk):
    """bf16 post-RoPE keys through T: transformed keys within 1e-3 relative
    error, code mismatch rate <= 1e-4 (boundary flips only), scales within
    one fp16 ulp, decode within tolerance."""
    import torch
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    T, TinvT = I.key_transforms(w, 3)
    T, TinvT = T[:2], TinvT[:2]
    n = 64 + 256 + 8 * 90
    cfg = wk.make_config(2, 2, 8, n + 8, bits=2)
    k, v = _kv(99, 2, n, 2)
    cache, oc = _append_both(wk, cfg, k, v, T, "bf16", [n - 2, 1, 1])
    ns, P, nr = oc.split()
    kr = H.rounded(k, "bf16").astype(np.float64)
    n_codes = n_bad = n_scale_bad = 0
    for u in range(4):
        b, h = divmod(u, 2)
        kt = kr[b, :, h] @ T[h].astype(np.float64).T          # exact k'
        ring = H.unit_window(cache, u, 0, "ring")[oc.recent_order()].astype(np.float64)
        want = kt[ns + P:]
        rel = np.linalg.norm(ring - want, axis=-1) / np.linalg.norm(want, axis=-1)
        assert rel.max() <= 1e-3
        codes = O.unpack_k_rows(H.unit_packed_planes(cache, u, 0, P), 2)
        n_codes += codes.size
        n_bad += int(np.sum(codes != oc.codes_k[u, :P]))
        gm = H.unit_meta(cache, u, 0, P)[:, 0].astype(np.float32)
        om = oc.meta_k[u, :P, 0].astype(np.float32)
        ulp = np.spacing(om.astype(np.float16)).astype(np.float32)
        assert np.all(np.abs(gm - om) <= ulp)
        n_scale_bad += int(np.sum(gm != om))
        # values are not transformed: bit-exact
        assert np.array_equal(H.unit_packed_planes(cache, u, 1, P)[0], oc.packed_v(u)[0])
    assert n_bad / n_codes <= 1e-4, (n_bad, n_codes)
    assert n_scale_bad / (4 * P) <= 0.02
    qd = torch.from_numpy(np.random.default_rng(1).standard_normal((2, 8, 128)).astype(np.float32))
    qp = wk.query_transform(qd.cuda(), torch.from_numpy(TinvT).cuda())
    out = cache.decode(qp).cpu().numpy()
    want = oc.decode(O.query_transform_gqa(qd.numpy(), TinvT.astype(np.float64)))
    assert H.rel_rms_err(out, want) <= DECODE_TOL


def test_error_paths(wk):
    import torch
    cfg = wk.make_config(1, 1, 4, 100)
    cache = wk.Cache(cfg)
    q = torch.zeros((1, 4, 128), device="cuda")
    with pytest.raises(wk.WushKVError) as e:
        cache.decode(q)
    assert e.value.status == wk.EINVAL
    k = torch.zeros((1, 101, 1, 128), device="cuda")
    with pytest.raises(wk.WushKVError) as e:
        cache.append(k, k)
    assert e.value.status == wk.ECAPACITY
    assert cache.tokens() == (0, 0, 0, 0)
    with pytest.raises(wk.WushKVError) as e:
        cache.append(k[:, :3].contiguous(), k[:, :3].contiguous(), bits=3)
    assert e.value.status == wk.EINVAL
    cache.append(k[:, :100].contiguous(), k[:, :100].contiguous())
    assert cache.tokens()[0] == 100
    with pytest.raises(wk.WushKVError):
        cache.append(k[:, :1].contiguous(), k[:, :1].contiguous())
    assert cache.layout().total_bytes == wk.cache_bytes(cfg)
