"""Shared helpers of the GPU parity tests: build the CUDA cache and the
oracle cache from the same seeded inputs and read raw device regions."""
from __future__ import annotations

import math

import numpy as np

from oracle import wushkv_oracle as O


def torch_dtype(name):
    import torch
    return {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[name]


def rounded(x: np.ndarray, name: str) -> np.ndarray:
    """float32 values after rounding to the input dtype (what both sides read)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch_dtype(name)).float().numpy()


def to_dev(x: np.ndarray, name: str):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch_dtype(name)).cuda().contiguous()


def region(cache, off: int, nbytes: int) -> np.ndarray:
    """Raw bytes [off, off + nbytes) of a cache buffer as uint8."""
    start = cache.base_ptr - cache.buffer.data_ptr() + off
    return cache.buffer[start:start + nbytes].cpu().numpy()


def _unit_blocks(cache, u: int, n_packed: int) -> np.ndarray:
    """Unit u's block records covering its first n_packed tokens, as
    [blocks][block_stride] uint8 (64 packed tokens per record)."""
    L = cache.layout()
    nb = (n_packed + 63) // 64
    return region(cache, u * L.unit_stride, nb * L.block_stride).reshape(nb, L.block_stride)


def unit_packed_planes(cache, u: int, kv: int, n_packed: int):
    """The packed plane bytes of unit u for its first n_packed tokens,
    gathered from the block records into uint32 arrays shaped like the
    oracle's pack_* output (token rows for 3- and 4-bit K, quads for 2-bit K
    and for V)."""
    L = cache.layout()
    blocks = _unit_blocks(cache, u, n_packed)
    out = []
    for p in range(L.n_planes):
        w = L.plane_bits[p]
        off = L.k_plane_off[p] if kv == 0 else L.v_plane_off[p]
        part = np.ascontiguousarray(blocks[:, off:off + 64 * 16 * w]).view(np.uint32)
        if kv == 0 and cache.cfg.bits == 2:
            # 2-bit K quads: 16 quads of 32 words per block record, in order
            out.append(part.reshape(-1, 32)[:n_packed // 4])
        elif kv == 0:
            # K rows sit at the swizzled position 8r + (j ^ (r & 3)) of token
            # 8r + j of each 64-token block
            rows = part.reshape(-1, 64, 4 * w)
            i = np.arange(64)
            pos = (i & ~7) | ((i & 7) ^ ((i >> 3) & 3))
            out.append(rows[:, pos].reshape(-1, 4 * w)[:n_packed])
        else:
            out.append(part.reshape(-1)[:n_packed * 4 * w].reshape(n_packed // 4, 16 * w))
    return out


def unit_meta(cache, u: int, kv: int, n_packed: int) -> np.ndarray:
    L = cache.layout()
    blocks = _unit_blocks(cache, u, n_packed)
    off = L.k_meta_off if kv == 0 else L.v_meta_off
    part = blocks[:, off:off + 64 * L.meta_bytes].reshape(-1)[:n_packed * L.meta_bytes]
    return np.ascontiguousarray(part).view(np.float16).reshape(n_packed, L.meta_bytes // 2)


def unit_window(cache, u: int, kv: int, which: str) -> np.ndarray:
    L = cache.layout()
    if which == "sink":
        off = (L.sink_k_off if kv == 0 else L.sink_v_off) + u * L.sink_unit_stride
        n = L.sink_unit_stride
    else:
        off = (L.ring_k_off if kv == 0 else L.ring_v_off) + u * L.ring_unit_stride
        n = L.ring_unit_stride
    return region(cache, off, n).view(np.float16).reshape(-1, 128)


def oracle_cfg(cfg) -> O.CacheConfig:
    return O.CacheConfig(batch=cfg.batch, n_kv_heads=cfg.n_kv_heads, n_q_heads=cfg.n_q_heads,
                         max_ctx=cfg.max_ctx, bits=cfg.bits, quantizer=cfg.quantizer,
                         sink=cfg.sink, recent=cfg.recent, chunk=cfg.chunk,
                         alpha=(cfg.quest_alpha or None), r_lo=cfg.clip_lo_rank,
                         r_hi=cfg.clip_hi_rank)


def compare_cache_bitexact(cache, oc: O.OracleCache, units=None):
    """Every byte of the packed planes, meta, sink and recent rows of the
    given units equals the oracle's."""
    ns, P, nr = oc.split()
    assert cache.tokens() == (oc.n, ns, P, nr)
    L = cache.layout()
    for u in (range(oc.cfg.units) if units is None else units):
        for kv in (0, 1):
            want = oc.packed_k(u) if kv == 0 else oc.packed_v(u)
            got = unit_packed_planes(cache, u, kv, P)
            for p in range(L.n_planes):
                assert np.array_equal(got[p], want[p]), (u, kv, p)
            meta = unit_meta(cache, u, kv, P)
            om = (oc.meta_k if kv == 0 else oc.meta_v)[u, :P, :meta.shape[1]]
            assert np.array_equal(meta.view(np.uint16), om.view(np.uint16)), (u, kv)
            sink = unit_window(cache, u, kv, "sink")[:ns]
            osink = (oc.sink_k if kv == 0 else oc.sink_v)[u, :ns]
            assert np.array_equal(sink.view(np.uint16), osink.view(np.uint16)), (u, kv)
            ring = unit_window(cache, u, kv, "ring")[oc.recent_order()]
            oring = (oc.ring_k if kv == 0 else oc.ring_v)[u, oc.recent_order()]
            assert np.array_equal(ring.view(np.uint16), oring.view(np.uint16)), (u, kv)
    check_guards(cache)


def rel_rms_err(got: np.ndarray, want: np.ndarray) -> float:
    """max |got - want| / RMS(want)."""
    return float(np.abs(got - want).max() / math.sqrt(float(np.mean(want ** 2))))


def check_unit_transformed(cache, oc: O.OracleCache, ou: int, T_h, k_h, u: int):
    """Unit u of the GPU cache against unit ou of an oracle cache fed the
    same rounded inputs, keys through T_h (k_h: that unit's post-RoPE keys).

    Bar: fp16 key windows within 1e-3 relative error of the exact k'; key
    codes mismatching on at most 1e-4 of elements (k' rounding-boundary
    flips); key scales within one fp16 ulp (QuEST) or two (affine: two
    independently rounded order statistics); value windows, codes and
    scales bit-exact."""
    ns, P, nr = oc.split()
    bits = oc.cfg.bits
    kt = np.asarray(k_h, np.float64) @ np.asarray(T_h, np.float64).T          # exact k'
    ring = unit_window(cache, u, 0, "ring")[oc.recent_order()].astype(np.float64)
    want = kt[ns + P:]
    rel = np.linalg.norm(ring - want, axis=-1) / np.linalg.norm(want, axis=-1)
    assert rel.max() <= 1e-3
    sink = unit_window(cache, u, 0, "sink")[:ns].astype(np.float64)
    rel = np.linalg.norm(sink - kt[:ns], axis=-1) / np.linalg.norm(kt[:ns], axis=-1)
    assert rel.max() <= 1e-3
    assert np.array_equal(unit_window(cache, u, 1, "ring")[oc.recent_order()].view(np.uint16),
                          oc.ring_v[ou, oc.recent_order()].view(np.uint16))
    assert np.array_equal(unit_window(cache, u, 1, "sink")[:ns].view(np.uint16),
                          oc.sink_v[ou, :ns].view(np.uint16))
    kc = O.unpack_k_rows(unit_packed_planes(cache, u, 0, P), bits)
    mism = float(np.mean(kc != oc.codes_k[ou, :P]))
    assert mism <= 1e-4, mism
    for p_, q_ in zip(unit_packed_planes(cache, u, 1, P), oc.packed_v(ou)):
        assert np.array_equal(p_, q_)
    gm = unit_meta(cache, u, 0, P).astype(np.float32)
    om = oc.meta_k[ou, :P, :gm.shape[1]].astype(np.float32)
    ulp = np.spacing(np.abs(om).astype(np.float16)).astype(np.float32)
    n_ulp = 1 if oc.cfg.quantizer == O.QUEST_INT else 2
    assert np.all(np.abs(gm - om) <= n_ulp * ulp)
    assert np.array_equal(unit_meta(cache, u, 1, P).view(np.uint16),
                          oc.meta_v[ou, :P, :gm.shape[1]].view(np.uint16))
    return mism


def check_guards(cache):
    """The guard bands after every cache region still hold their fill byte
    (no kernel wrote past a region)."""
    from bit_kv_cache_post_b200 import wushkv as wk
    for off in cache.guard_offsets():
        band = region(cache, off, wk.GUARD_BYTES)
        assert np.all(band == wk.GUARD_FILL), ("guard band written", off)


def unit_state_from_export(cache, b: int, h: int):
    """(K, V) of unit (b, h) as the GPU cache holds them, read through
    wushkv_export and dequantised with the oracle's reconstruction rules:
    fp16 rows for window tokens, (codes, scales) for packed ones."""
    cfg = cache.cfg
    n = cache.tokens(b)[0]
    out = []
    for kv in (0, 1):
        codes, meta, rows, kinds = cache.export(b, h, kv, 0, n)
        x = rows.view(np.float16).astype(np.float64)
        pk = kinds == 1
        if pk.any():
            m = meta[pk].view(np.float16)
            if cfg.quantizer == O.QUEST_INT:
                x[pk] = O.quest_dequantize(codes[pk], m[:, 0], cfg.bits)
            else:
                x[pk] = O.affine_dequantize(codes[pk], m[:, 0], m[:, 1])
        out.append(x)
    return out[0], out[1]


def compare_unit_by_export(cache, b: int, h: int, oc: O.OracleCache, ou: int):
    """Unit (b, h) of the GPU cache, read through wushkv_export, equals unit
    ou of the oracle cache bit for bit: kinds, fp16 window rows, packed
    codes and scales of K and V."""
    cfg = cache.cfg
    n = cache.tokens(b)[0]
    ns, P, nr = oc.split()
    assert (n, ns, P, nr) == (oc.n, *oc.split())
    W = cfg.recent + cfg.chunk
    nm = 2 if cfg.quantizer == O.AFFINE_PCTCLIP else 1
    for kv in (0, 1):
        codes, meta, rows, kinds = cache.export(b, h, kv, 0, n)
        sink = oc.sink_k if kv == 0 else oc.sink_v
        ring = oc.ring_k if kv == 0 else oc.ring_v
        ocodes = oc.codes_k if kv == 0 else oc.codes_v
        ometa = oc.meta_k if kv == 0 else oc.meta_v
        assert np.array_equal(kinds, np.array([0] * ns + [1] * P + [2] * nr, np.int8)), (b, h, kv)
        assert np.array_equal(rows[:ns], sink[ou, :ns].view(np.uint16)), (b, h, kv)
        slots = [(t - cfg.sink) % W for t in range(ns + P, n)]
        assert np.array_equal(rows[ns + P:], ring[ou, slots].view(np.uint16)), (b, h, kv)
        assert np.array_equal(codes[ns:ns + P], ocodes[ou, :P]), (b, h, kv)
        assert np.array_equal(meta[ns:ns + P, :nm], ometa[ou, :P, :nm].view(np.uint16)), (b, h, kv)
