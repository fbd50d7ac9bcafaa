"""Plain CPU oracle for the WUSH-KV online cache path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
table or constant generator with the CUDA library; the two agree only on the
byte format of the packed cache, which each side writes out on its own.

Sources (web pages about arXiv 2609.38121, "WUSH-KV: KV Cache Quantization
with Data-Adaptive Transforms"):

* [ai-papers-daily] slinene.github.io summary "WUSH-KV：数据自适应变换的 KV Cache
  低比特量化", sections 工作参考价值 (practical value) and 方法关键点
  (method key points).
* [secrett2633] blog.secrett2633 review "[논문리뷰] WUSH-KV: ...", section
  "1. Key Terms & Definitions", entry "QuEST Quantizer".
* [weekinpapers] weekinpapers.com "Kv cache quantization reduces memory for
  long context language models", Abstract.

What the pages fix, and what this file therefore computes:

* Each KV head has an invertible d x d key transform; it acts on keys after
  RoPE, one d x d product per new token, and the query side uses the inverse
  transpose so that q'.k' = q.k ([ai-papers-daily] 方法关键点, 3rd bullet;
  工作参考价值, 2nd bullet).  Values arrive already transformed because the
  value transform is folded into W_V / W_O (same bullet), so V is used as
  given.
* Quantisation is per token; QuEST INT scales by the token's RMS and
  reconstructs at bin centres ([secrett2633] Key Terms, QuEST entry); the
  serving variant is a percentile-clipped affine quantiser
  ([ai-papers-daily] 方法关键点, 4th bullet; [weekinpapers] Abstract).
* The first 64 (sink) tokens and the latest 256 (recent) tokens stay in fp16
  and the recent window is flushed to the quantised cache in chunks of 8 or
  16 ([ai-papers-daily] 工作参考价值 3rd bullet, 方法关键点 5th bullet).
* Attention is grouped-query attention ([secrett2633] Key Terms, GQA entry).

Everything else is a reading of silent or ambiguous text; each reading is
named where it is used (``READING:``) and collected in the design notes.

Floating point: transforms and attention run in float64.  The quantisers
follow an exact float32 specification so that the integer codes they decide
are reproducible bit for bit by an independent implementation.

Parity status: every function below is pinned by ``tests/test_oracle_*.py``
except the numeric value of the QuEST clip ratio alpha_b as the paper's
authors use it, which the pages never state ("parity unpinned" for that
value; its Gaussian-MSE optimality, the reading taken, is pinned against
Max's published table).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128

QUEST_INT = 0
AFFINE_PCTCLIP = 1


# ---------------------------------------------------------------------------
# Transforms ([ai-papers-daily] 方法关键点, 3rd bullet)
# ---------------------------------------------------------------------------

def transform_keys(k: np.ndarray, T: np.ndarray) -> np.ndarray:
    """k' = T k for every key vector (last axis), float64.

    ``T`` is d x d row-major: k'_i = sum_j T[i, j] k_j.  Applied after RoPE.
    """
    k64 = np.asarray(k, dtype=np.float64)
    return k64 @ np.asarray(T, dtype=np.float64).T


def transform_query(q: np.ndarray, T_invT: np.ndarray) -> np.ndarray:
    """q' = T^{-T} q for every query vector (last axis), float64.

    ``T_invT`` is the inverse transpose of the key transform, given as an
    input (the calibration that builds T is offline and out of scope).
    """
    q64 = np.asarray(q, dtype=np.float64)
    return q64 @ np.asarray(T_invT, dtype=np.float64).T


def query_transform_gqa(q: np.ndarray, T_invT: np.ndarray) -> np.ndarray:
    """q'[b, h] = T_invT[h // G] q[b, h] for q of shape [B, Hq, d].

    READING (GQA map): query head h reads KV head floor(h / G), G = Hq/Hkv,
    i.e. contiguous groups -- the pages name GQA but not the grouping.
    """
    q64 = np.asarray(q, dtype=np.float64)
    B, Hq, d = q64.shape
    Hkv = T_invT.shape[0]
    G = Hq // Hkv
    out = np.empty_like(q64)
    for h in range(Hq):
        out[:, h, :] = transform_query(q64[:, h, :], T_invT[h // G])
    return out


# ---------------------------------------------------------------------------
# Window policy ([ai-papers-daily] 工作参考价值 3rd bullet; 方法关键点 5th)
# ---------------------------------------------------------------------------

def window_split(n: int, sink: int, recent: int, chunk: int) -> tuple[int, int, int]:
    """(n_sink, n_packed, n_recent) for a sequence holding ``n`` tokens.

    READING: tokens [0, min(n, sink)) are fp16 sink tokens.  Later tokens
    enter the fp16 recent window first; whenever the window holds at least
    recent + chunk tokens, its oldest ``chunk`` tokens are quantised and
    moved to the packed cache.  So at least ``recent`` tokens are always
    fp16 once that many exist, and the result depends only on ``n``.
    """
    n_sink = min(n, sink)
    m = n - n_sink
    packed = chunk * ((m - recent) // chunk) if m >= recent + chunk else 0
    return n_sink, packed, m - packed


def ring_slot(token: int, sink: int, recent: int, chunk: int) -> int:
    """Ring position of a post-sink token in the recent window."""
    return (token - sink) % (recent + chunk)


# ---------------------------------------------------------------------------
# QuEST INT clip ratio
# ---------------------------------------------------------------------------

def _phi(x: float) -> float:
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi(x: float) -> float:
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _prim_m0(x: float) -> float:
    """Primitive of phi: Phi(x), with the limits at +-inf."""
    if x == math.inf:
        return 1.0
    if x == -math.inf:
        return 0.0
    return _Phi(x)


def _prim_m1(x: float) -> float:
    """Primitive of x phi(x): -phi(x) (zero at +-inf)."""
    return 0.0 if math.isinf(x) else -_phi(x)


def _prim_m2(x: float) -> float:
    """Primitive of x^2 phi(x): Phi(x) - x phi(x)."""
    if math.isinf(x):
        return _prim_m0(x)
    return _Phi(x) - x * _phi(x)


def _second_moment(a: float, b: float, c: float) -> float:
    """Integral over [a, b] of (x - c)^2 phi(x) dx, unit Gaussian phi."""
    m2 = _prim_m2(b) - _prim_m2(a)
    m1 = _prim_m1(b) - _prim_m1(a)
    m0 = _prim_m0(b) - _prim_m0(a)
    return m2 - 2.0 * c * m1 + c * c * m0


def _first_moment(a: float, b: float, c: float) -> float:
    """Integral over [a, b] of (x - c) phi(x) dx."""
    return (_prim_m1(b) - _prim_m1(a)) - c * (_prim_m0(b) - _prim_m0(a))


def _bins(alpha: float, levels: int):
    step = 2.0 * alpha / levels
    for i in range(-levels // 2, levels // 2):
        lo = -math.inf if i == -levels // 2 else i * step
        hi = math.inf if i == levels // 2 - 1 else (i + 1) * step
        yield i, lo, hi, (i + 0.5) * step


def uniform_gaussian_mse(alpha: float, levels: int) -> float:
    """Mean squared error of the L-level mid-rise uniform quantiser with
    clip range [-alpha, alpha] applied to X ~ N(0, 1).

    Levels sit at (i + 1/2) * step for i in [-L/2, L/2), step = 2 alpha / L;
    inputs beyond the range map to the end levels.
    """
    return sum(_second_moment(lo, hi, c) for _, lo, hi, c in _bins(alpha, levels))


def uniform_gaussian_mse_deriv(alpha: float, levels: int) -> float:
    """d MSE / d alpha.  Interior cell edges sit midway between levels, so
    their movement contributes nothing; only the levels move, at rate
    dc_i/dalpha = (2i + 1) / L."""
    return sum(-2.0 * ((2 * i + 1) / levels) * _first_moment(lo, hi, c)
               for i, lo, hi, c in _bins(alpha, levels))


def quest_alpha(bits: int) -> float:
    """Clip ratio alpha_b: clip range = +-alpha_b * RMS of the token.

    READING: the pages name QuEST INT ("RMS-based scale, bin-centre
    reconstruction", [secrett2633] Key Terms) but give no clip ratio.  We take
    the ratio that minimises the exact mean squared error of the 2^b-level
    uniform quantiser on a unit Gaussian (the classic optimum of Max, 1960):
    the zero of d MSE / d alpha, found by bisection to float64 resolution.
    """
    levels = 1 << bits
    a, b = 0.25, 16.0
    assert uniform_gaussian_mse_deriv(a, levels) < 0 < uniform_gaussian_mse_deriv(b, levels)
    for _ in range(200):
        mid = 0.5 * (a + b)
        if mid in (a, b):
            break
        if uniform_gaussian_mse_deriv(mid, levels) < 0:
            a = mid
        else:
            b = mid
    return 0.5 * (a + b)


# ---------------------------------------------------------------------------
# Per-token quantisers: exact float32 specification
# ---------------------------------------------------------------------------

def to_fp16_values(x: np.ndarray) -> np.ndarray:
    """Round to fp16 (round-to-nearest-even) and return the values as float32.

    READING: the recent window stores fp16 vectors and the packed cache is
    filled by flushing that window, so every vector is quantised from its
    fp16-rounded value.  Prefill tokens go through the same rounding so the
    cache state depends only on the token count.
    """
    return np.asarray(x).astype(np.float16).astype(np.float32)


def quest_quantize(x: np.ndarray, bits: int, alpha: float):
    """QuEST INT on each row of ``x`` (float32 values, last axis = 128).

    Returns (codes uint8/uint16 [.., 128], delta float16 [..]).

    [secrett2633] Key Terms (QuEST entry): scale from the token's RMS,
    reconstruction at bin centres, per token.  READINGS for what the page
    leaves open:
      * symmetric mid-rise grid of L = 2^b levels at (i + 1/2) * delta,
        i in [-L/2, L/2), so the clip range is +-alpha * RMS with
        delta = alpha * RMS / 2^(b-1);
      * ss = sum of squares in float64 (squares of float32 values are exact
        there), rms = sqrt(ss / 128) in float64, delta rounded once from
        float64 to fp16 (the stored scale);
      * inv = RN32(1 / delta_h); t = RN32(RN32(x * inv) + L/2);
        code = clamp(floor(t), 0, L - 1);
      * delta_h == 0 (all-zero token): every code is L/2 and reconstructs
        to 0.
    """
    x32 = np.asarray(x, dtype=np.float32)
    L = 1 << bits
    ss = np.sum(x32.astype(np.float64) ** 2, axis=-1)
    rms = np.sqrt(ss / float(x32.shape[-1]))
    delta_h = (alpha * rms / float(1 << (bits - 1))).astype(np.float16)
    d32 = delta_h.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (np.float32(1.0) / d32).astype(np.float32)
        t = (x32 * inv[..., None]).astype(np.float32)
        t = (t + np.float32(L // 2)).astype(np.float32)
    zero = (d32 == 0)[..., None]
    t = np.where(zero, np.float32(L // 2), t)
    codes = np.clip(np.floor(t), 0, L - 1).astype(np.uint16 if bits > 8 else np.uint8)
    return codes, delta_h


def quest_dequantize(codes: np.ndarray, delta_h: np.ndarray, bits: int) -> np.ndarray:
    """x_hat = (code - L/2 + 1/2) * delta, float64 (bin centre)."""
    L = 1 << bits
    return (codes.astype(np.float64) - L / 2 + 0.5) * delta_h.astype(np.float64)[..., None]


def affine_quantize(x: np.ndarray, bits: int, r_lo: int, r_hi: int):
    """Percentile-clipped affine quantiser on each row of ``x``.

    Returns (codes [.., 128], scale float16 [..], lo float16 [..]).

    [ai-papers-daily] 方法关键点 4th bullet and [weekinpapers] Abstract name an
    OSCAR-style percentile-clipped affine quantiser without its details.
    READINGS:
      * lo, hi = the r_lo-th and r_hi-th smallest of the token's 128 values
        (1-indexed order statistics; ties are harmless because order
        statistics are values);
      * lo_h = fp16(lo); s_h = fp16(RN32(RN32(hi - lo) / (L - 1)));
      * inv = RN32(1 / s_h); t = RN32(RN32(x - lo_h) * inv);
        code = clamp(round-half-even(t), 0, L - 1);
      * x_hat = lo_h + code * s_h;  s_h == 0 gives code 0 everywhere.
    """
    x32 = np.asarray(x, dtype=np.float32)
    L = 1 << bits
    srt = np.sort(x32, axis=-1)
    lo = srt[..., r_lo - 1]
    hi = srt[..., r_hi - 1]
    lo_h = lo.astype(np.float16)
    rng = (hi - lo).astype(np.float32)
    s32 = (rng / np.float32(L - 1)).astype(np.float32)
    s_h = s32.astype(np.float16)
    sd = s_h.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (np.float32(1.0) / sd).astype(np.float32)
        t = (x32 - lo_h.astype(np.float32)[..., None]).astype(np.float32)
        t = (t * inv[..., None]).astype(np.float32)
    t = np.where((sd == 0)[..., None], np.float32(0.0), t)
    codes = np.clip(np.rint(t), 0, L - 1).astype(np.uint16 if bits > 8 else np.uint8)
    return codes, s_h, lo_h


def affine_dequantize(codes: np.ndarray, s_h: np.ndarray, lo_h: np.ndarray) -> np.ndarray:
    """x_hat = lo + code * s, float64."""
    return (lo_h.astype(np.float64)[..., None]
            + codes.astype(np.float64) * s_h.astype(np.float64)[..., None])


# ---------------------------------------------------------------------------
# Packed byte format.  The pages give no layout ("low-bit" only), so this is
# the library's documented format, restated here from its definition:
#
#   planes: 2-bit codes -> one 2-bit plane; 4-bit -> one 4-bit plane;
#           3-bit -> a 2-bit plane of (code & 3) then a 1-bit plane of
#           (code >> 2).  A plane of width w packs P = 8 / w fields in each
#           byte; field s of byte beta of a 32-bit little-endian word sits at
#           bit 8*beta + w*s.
#   K rows, 3 and 4 bits (one token, 128 dims, 4w words per plane): for c in
#     0..3, h in 0..1, ks in 0..3, beta in 0..3, rho = 4h + ks:
#       word = c*w + rho // P, field s = rho % P, dim = 32ks + 4c + 16h + beta.
#   K quads, 2 bits (4 consecutive tokens, 32 words): word omega holds dims
#     4 omega + beta at byte beta, and token 4*quad + f at field f; with
#     omega = 8ks + 4h + c it is stored at position
#     4 ((2c + ks // 2) xor (quad mod 2)) + 2 (ks mod 2) + h of the quad.
#   V quads (4 consecutive tokens, 8*2w words per plane): for r in 0..7,
#     rho in 0..15 (mt = rho // 2, rh = rho % 2), beta in 0..3:
#       unit word j = rho // P, field s = rho % P,
#       dim = 16mt + r + 8rh, token = 4*quad + beta.
#     The 2w words of row unit r are stored at unit position
#     pos = (r + 2*(quad mod 4)) mod 8 of the quad: w = 1 -> words 2pos + j;
#     w = 2 -> words 4pos + j; w = 4 -> words 4pos + j for j < 4 and
#     32 + 4pos + (j - 4) for j >= 4.  (quad = quad index within the unit.)
# ---------------------------------------------------------------------------

def plane_widths(bits: int) -> list[int]:
    return {2: [2], 3: [2, 1], 4: [4]}[bits]


def _plane_values(codes: np.ndarray, bits: int) -> list[np.ndarray]:
    c = codes.astype(np.uint32)
    if bits == 3:
        return [c & 3, c >> 2]
    return [c]


def k2_word_pos(quad: int, omega: int) -> int:
    """Position of word omega (dims 4 omega .. 4 omega + 3) in a 2-bit K quad."""
    ks, h, c = omega // 8, (omega // 4) % 2, omega % 4
    return 4 * ((2 * c + ks // 2) ^ (quad % 2)) + 2 * (ks % 2) + h


def pack_k_rows(codes: np.ndarray, bits: int) -> list[np.ndarray]:
    """codes [N, 128] -> one uint32 array per plane: [N, 4w] token rows at 3
    and 4 bits; [N / 4, 32] quads at 2 bits (N a multiple of 4)."""
    if bits == 2:
        n = codes.shape[0]
        assert n % 4 == 0, "2-bit K codes are packed in quads of 4 tokens"
        c = codes.astype(np.uint32).reshape(n // 4, 4, HEAD_DIM)
        words = np.zeros((n // 4, 32), dtype=np.uint32)
        for q in range(n // 4):
            for omega in range(32):
                wd = np.uint32(0)
                for beta in range(4):
                    for f in range(4):
                        wd |= c[q, f, 4 * omega + beta] << np.uint32(8 * beta + 2 * f)
                words[q, k2_word_pos(q, omega)] = wd
        return [words]
    out = []
    for w, vals in zip(plane_widths(bits), _plane_values(codes, bits)):
        P = 8 // w
        words = np.zeros(codes.shape[:-1] + (4 * w,), dtype=np.uint32)
        for c in range(4):
            for h in range(2):
                for ks in range(4):
                    rho = 4 * h + ks
                    word, s = c * w + rho // P, rho % P
                    for beta in range(4):
                        dim = 32 * ks + 4 * c + 16 * h + beta
                        words[..., word] |= vals[..., dim] << np.uint32(8 * beta + w * s)
        out.append(words)
    return out


def unpack_k_rows(planes: list[np.ndarray], bits: int) -> np.ndarray:
    """Inverse of :func:`pack_k_rows`: -> codes [N, 128]."""
    if bits == 2:
        words = planes[0]
        nq = words.shape[0]
        codes = np.zeros((nq, 4, HEAD_DIM), dtype=np.uint32)
        for q in range(nq):
            for omega in range(32):
                wd = words[q, k2_word_pos(q, omega)]
                for beta in range(4):
                    for f in range(4):
                        codes[q, f, 4 * omega + beta] = (wd >> np.uint32(8 * beta + 2 * f)) & np.uint32(3)
        return codes.reshape(nq * 4, HEAD_DIM).astype(np.uint8)
    n = planes[0].shape[:-1]
    codes = np.zeros(n + (HEAD_DIM,), dtype=np.uint32)
    shift = 0
    for w, words in zip(plane_widths(bits), planes):
        P, mask = 8 // w, np.uint32((1 << w) - 1)
        for c in range(4):
            for h in range(2):
                for ks in range(4):
                    rho = 4 * h + ks
                    word, s = c * w + rho // P, rho % P
                    for beta in range(4):
                        dim = 32 * ks + 4 * c + 16 * h + beta
                        f = (words[..., word] >> np.uint32(8 * beta + w * s)) & mask
                        codes[..., dim] |= f << np.uint32(shift)
        shift += w
    return codes.astype(np.uint8)


def v_word_index(quad: int, r: int, j: int, w: int) -> int:
    """Flat word index in a V quad of unit word j of row unit r."""
    pos = (r + 2 * (quad % 4)) % 8
    if w == 4:
        return 4 * pos + j if j < 4 else 32 + 4 * pos + (j - 4)
    return 2 * w * pos + j


def pack_v_quads(codes: np.ndarray, bits: int) -> list[np.ndarray]:
    """codes [NQ, 4, 128] (4 consecutive tokens per quad; quad index = first
    axis) -> one uint32 array [NQ, 16w] per plane."""
    out = []
    nq = codes.shape[0]
    for w, vals in zip(plane_widths(bits), _plane_values(codes, bits)):
        P = 8 // w
        unit = np.zeros((nq, 8, 2 * w), dtype=np.uint32)
        for r in range(8):
            for rho in range(16):
                mt, rh = rho // 2, rho % 2
                dim = 16 * mt + r + 8 * rh
                word, s = rho // P, rho % P
                for beta in range(4):
                    unit[:, r, word] |= vals[:, beta, dim] << np.uint32(8 * beta + w * s)
        words = np.zeros((nq, 16 * w), dtype=np.uint32)
        for q in range(nq):
            for r in range(8):
                for j in range(2 * w):
                    words[q, v_word_index(q, r, j, w)] = unit[q, r, j]
        out.append(words)
    return out


def unpack_v_quads(planes: list[np.ndarray], bits: int) -> np.ndarray:
    """Inverse of :func:`pack_v_quads`: -> codes [NQ, 4, 128]."""
    nq = planes[0].shape[0]
    codes = np.zeros((nq, 4, HEAD_DIM), dtype=np.uint32)
    shift = 0
    for w, flat in zip(plane_widths(bits), planes):
        P, mask = 8 // w, np.uint32((1 << w) - 1)
        words = np.zeros((nq, 8, 2 * w), dtype=np.uint32)
        for q in range(nq):
            for r in range(8):
                for j in range(2 * w):
                    words[q, r, j] = flat[q, v_word_index(q, r, j, w)]
        for r in range(8):
            for rho in range(16):
                mt, rh = rho // 2, rho % 2
                dim = 16 * mt + r + 8 * rh
                word, s = rho // P, rho % P
                for beta in range(4):
                    f = (words[:, r, word] >> np.uint32(8 * beta + w * s)) & mask
                    codes[:, beta, dim] |= f << np.uint32(shift)
        shift += w
    return codes.astype(np.uint8)


# ---------------------------------------------------------------------------
# Attention (float64)
# ---------------------------------------------------------------------------

def attention_f64(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q K^T) V for q [G, d], K [n, d], V [n, d] (float64).

    Softmax with the row maximum subtracted before exponentiation.
    """
    q64 = np.atleast_2d(np.asarray(q, dtype=np.float64))
    s = scale * (q64 @ np.asarray(K, dtype=np.float64).T)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ np.asarray(V, dtype=np.float64)


# ---------------------------------------------------------------------------
# The cache: append (transform -> windows -> quantise on flush) and decode
# ---------------------------------------------------------------------------

@dataclass
class CacheConfig:
    batch: int
    n_kv_heads: int
    n_q_heads: int
    max_ctx: int
    bits: int = 2
    quantizer: int = QUEST_INT
    sink: int = 64
    recent: int = 256
    chunk: int = 8
    alpha: float | None = None     # None -> quest_alpha(bits)
    r_lo: int = 2
    r_hi: int = 127

    @property
    def units(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def quest_alpha_value(self) -> float:
        return quest_alpha(self.bits) if self.alpha is None else float(self.alpha)


class OracleCache:
    """One layer's cache for ``batch`` sequences x ``n_kv_heads`` heads.

    Unit u = b * n_kv_heads + h.  Codes are kept unpacked in natural dim
    order; :meth:`packed_k` / :meth:`packed_v` produce the byte format.
    """

    def __init__(self, cfg: CacheConfig):
        self.cfg = cfg
        U, d = cfg.units, HEAD_DIM
        W = cfg.recent + cfg.chunk
        self.sink_k = np.zeros((U, cfg.sink, d), np.float16)
        self.sink_v = np.zeros((U, cfg.sink, d), np.float16)
        self.ring_k = np.zeros((U, W, d), np.float16)
        self.ring_v = np.zeros((U, W, d), np.float16)
        cap = cfg.max_ctx
        self.codes_k = np.zeros((U, cap, d), np.uint8)
        self.codes_v = np.zeros((U, cap, d), np.uint8)
        # QuEST: meta[..., 0] = delta.  Affine: meta[..., 0] = s, [..., 1] = lo.
        self.meta_k = np.zeros((U, cap, 2), np.float16)
        self.meta_v = np.zeros((U, cap, 2), np.float16)
        self.n = 0
        self.n_packed = 0

    # -- quantiser dispatch -------------------------------------------------
    def _quantize(self, x16: np.ndarray):
        cfg = self.cfg
        x = x16.astype(np.float32)
        meta = np.zeros(x.shape[:-1] + (2,), np.float16)
        if cfg.quantizer == QUEST_INT:
            codes, delta = quest_quantize(x, cfg.bits, cfg.quest_alpha_value())
            meta[..., 0] = delta
        else:
            codes, s, lo = affine_quantize(x, cfg.bits, cfg.r_lo, cfg.r_hi)
            meta[..., 0], meta[..., 1] = s, lo
        return codes, meta

    def _dequantize(self, codes: np.ndarray, meta: np.ndarray) -> np.ndarray:
        if self.cfg.quantizer == QUEST_INT:
            return quest_dequantize(codes, meta[..., 0], self.cfg.bits)
        return affine_dequantize(codes, meta[..., 0], meta[..., 1])

    # -- append ---------------------------------------------------------------
    def append(self, k: np.ndarray, v: np.ndarray, T: np.ndarray | None):
        """Append ``n_tok`` tokens to every sequence.

        k, v: [B, n_tok, Hkv, 128].  With ``T`` ([Hkv, 128, 128]) the keys are
        post-RoPE keys and are transformed in float64, then rounded once to
        fp16.  With ``T`` None the keys are taken as already transformed and
        rounded from their own dtype to fp16 (the float32 bit-exact entry).
        """
        cfg = self.cfg
        B, n_tok, Hkv, d = k.shape
        if self.n + n_tok > cfg.max_ctx:
            raise ValueError("capacity exceeded")
        if T is not None:
            kt = np.empty((B, n_tok, Hkv, d), np.float64)
            for h in range(Hkv):
                kt[:, :, h, :] = transform_keys(k[:, :, h, :], T[h])
            k16 = kt.astype(np.float16)           # float64 -> fp16 directly
        else:
            k16 = np.asarray(k).astype(np.float16)
        v16 = np.asarray(v).astype(np.float16)
        # unit-major views [U, n_tok, d]
        k16 = k16.transpose(0, 2, 1, 3).reshape(B * Hkv, n_tok, d)
        v16 = v16.transpose(0, 2, 1, 3).reshape(B * Hkv, n_tok, d)
        S, R, C = cfg.sink, cfg.recent, cfg.chunk
        W = R + C
        for i in range(n_tok):
            t = self.n
            if t < S:
                self.sink_k[:, t] = k16[:, i]
                self.sink_v[:, t] = v16[:, i]
            else:
                slot = ring_slot(t, S, R, C)
                self.ring_k[:, slot] = k16[:, i]
                self.ring_v[:, slot] = v16[:, i]
                count = t + 1 - S - self.n_packed
                if count >= W:
                    first = S + self.n_packed
                    slots = [ring_slot(first + j, S, R, C) for j in range(C)]
                    P = self.n_packed
                    ck, mk = self._quantize(self.ring_k[:, slots])
                    cv, mv = self._quantize(self.ring_v[:, slots])
                    self.codes_k[:, P:P + C], self.meta_k[:, P:P + C] = ck, mk
                    self.codes_v[:, P:P + C], self.meta_v[:, P:P + C] = cv, mv
                    self.n_packed += C
            self.n += 1
        assert window_split(self.n, S, R, C)[1] == self.n_packed

    # -- state views ------------------------------------------------------------
    def split(self) -> tuple[int, int, int]:
        c = self.cfg
        return window_split(self.n, c.sink, c.recent, c.chunk)

    def recent_order(self) -> list[int]:
        """Ring slots of the recent tokens, oldest first."""
        c = self.cfg
        ns, P, nr = self.split()
        first = ns + P
        return [ring_slot(first + j, c.sink, c.recent, c.chunk) for j in range(nr)]

    def unit_kv(self, u: int) -> tuple[np.ndarray, np.ndarray]:
        """All cached keys and values of unit ``u`` in token order, float64
        (fp16 windows widened exactly; packed tokens dequantised)."""
        ns, P, nr = self.split()
        order = self.recent_order()
        K = np.concatenate([
            self.sink_k[u, :ns].astype(np.float64),
            self._dequantize(self.codes_k[u, :P], self.meta_k[u, :P]),
            self.ring_k[u, order].astype(np.float64)])
        V = np.concatenate([
            self.sink_v[u, :ns].astype(np.float64),
            self._dequantize(self.codes_v[u, :P], self.meta_v[u, :P]),
            self.ring_v[u, order].astype(np.float64)])
        return K, V

    def packed_k(self, u: int) -> list[np.ndarray]:
        P = self.n_packed
        return pack_k_rows(self.codes_k[u, :P], self.cfg.bits)

    def packed_v(self, u: int) -> list[np.ndarray]:
        P = self.n_packed
        return pack_v_quads(self.codes_v[u, :P].reshape(P // 4, 4, HEAD_DIM), self.cfg.bits)

    # -- decode -----------------------------------------------------------------
    def decode(self, q_prime: np.ndarray, scale: float | None = None,
               units: list[int] | None = None) -> np.ndarray:
        """GQA decode attention of q' [B, Hq, 128] over the whole cache.

        READINGS: scale defaults to 1/sqrt(128); the output stays in the
        transformed value space (the caller's W_O carries the inverse value
        transform); the query attends to the cache after its own token was
        appended.  ``units`` restricts the work to some (b, h) units; other
        outputs are left NaN.
        """
        cfg = self.cfg
        if scale is None:
            scale = 1.0 / math.sqrt(HEAD_DIM)
        B, Hq, d = q_prime.shape
        G = cfg.group
        out = np.full((B, Hq, d), np.nan)
        for u in (range(cfg.units) if units is None else units):
            b, h = divmod(u, cfg.n_kv_heads)
            K, V = self.unit_kv(u)
            out[b, h * G:(h + 1) * G] = attention_f64(q_prime[b, h * G:(h + 1) * G], K, V, scale)
        return out


    def prefill_attention(self, q_prime: np.ndarray, scale: float | None = None,
                          units: list[int] | None = None) -> np.ndarray:
        """Causal attention of a chunk of queries over the cache (chunked
        prefill), q' [B, n_q, Hq, 128] -> [B, n_q, Hq, 128].

        READING (the pages describe no prefill attention; this is the plain
        reading that the decode's rules give): the chunk's tokens are the last
        n_q tokens of every sequence and have been appended first; the query
        of token p = n - n_q + i attends to tokens 0 .. p as the cache holds
        them (fp16 windows, dequantised packed tokens), just as a decode query
        attends after its own token was appended.  ``units`` restricts the
        work; other outputs are left NaN.
        """
        cfg = self.cfg
        if scale is None:
            scale = 1.0 / math.sqrt(HEAD_DIM)
        B, nq, Hq, d = q_prime.shape
        G = cfg.group
        n = self.n
        out = np.full((B, nq, Hq, d), np.nan)
        for u in (range(cfg.units) if units is None else units):
            b, h = divmod(u, cfg.n_kv_heads)
            K, V = self.unit_kv(u)
            for i in range(nq):
                p = n - nq + i
                out[b, i, h * G:(h + 1) * G] = attention_f64(q_prime[b, i, h * G:(h + 1) * G],
                                                             K[:p + 1], V[:p + 1], scale)
        return out


# ---------------------------------------------------------------------------
# Module-output error (summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化",
# 关键实验, first bullet: the relative error of the attention module's output
# with the quantised cache, summarised by a geometric mean; the pages report it
# for 2-bit caches on real model data).  READING: per (sequence, query head),
# e = ||o_q - o|| / ||o|| where o is exact float64 attention over the keys and
# values as given and o_q the decode output over the quantised cache built
# with transform T; the summary is exp(mean(log e)).
# ---------------------------------------------------------------------------

def output_errors(k: np.ndarray, v: np.ndarray, q: np.ndarray, T: np.ndarray, TinvT: np.ndarray,
                  cfg: CacheConfig) -> np.ndarray:
    """Relative output error per (sequence, query head) of one decode query
    per head after appending all of k, v ([B, n, Hkv, 128]) through T;
    q [B, Hq, 128].  Returns [B, Hq]."""
    B, n, Hkv, d = k.shape
    oc = OracleCache(cfg)
    oc.append(k, v, np.asarray(T, np.float64))
    qp = query_transform_gqa(q, np.asarray(TinvT, np.float64))
    got = oc.decode(qp)
    G = cfg.group
    scale = 1.0 / math.sqrt(HEAD_DIM)
    err = np.empty((B, q.shape[1]))
    for b in range(B):
        for h in range(Hkv):
            ref = attention_f64(q[b, h * G:(h + 1) * G], k[b, :, h], v[b, :, h], scale)
            diff = got[b, h * G:(h + 1) * G] - ref
            err[b, h * G:(h + 1) * G] = np.linalg.norm(diff, axis=-1) / np.linalg.norm(ref, axis=-1)
    return err


def geometric_mean(x: np.ndarray) -> float:
    return float(np.exp(np.mean(np.log(np.asarray(x, np.float64)))))
