"""Pins of the CPU oracle against things other than itself.

Each ``check_*`` takes the oracle's functions as arguments so that
``test_oracle_mutations.py`` can hand it a copy with a planted mistake and
watch the check fail.  The checks use closed forms, published tables, brute
force on tiny inputs (``oracle.brute``), invariants of the mathematics and the
window counts of the summary page -- never a retyped copy of the oracle's own
formula.
"""
from __future__ import annotations

import math
import os

import numpy as np

from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([float(v) for v in line.split()])
    return rows


# --- QuEST clip ratio ---------------------------------------------------------

def check_alpha_max_table(quest_alpha, mse):
    """alpha_b reproduces Max (1960): optimum uniform step and its MSE."""
    for levels, step, err in _table("max1960_uniform_gaussian.txt"):
        bits = int(round(math.log2(levels)))
        a = quest_alpha(bits)
        got_step = 2.0 * a / levels
        assert abs(got_step - step) <= 6e-4 * step, (levels, got_step, step)
        got_mse = mse(a, int(levels))
        assert abs(got_mse - err) <= 1e-3 * err + 5e-6, (levels, got_mse, err)


def check_mse_monte_carlo(mse, seed=0):
    """The closed-form MSE matches a direct simulation of the quantiser."""
    g = np.random.default_rng(seed)
    x = g.standard_normal(400_000)
    for levels, alpha in ((4, 2.0), (8, 2.3), (16, 3.1)):
        step = 2 * alpha / levels
        idx = np.clip(np.floor(x / step), -levels // 2, levels // 2 - 1)
        emp = np.mean((x - (idx + 0.5) * step) ** 2)
        assert abs(emp - mse(alpha, levels)) < 0.02 * emp


# --- QuEST INT ------------------------------------------------------------------

def check_quest_brute(quest_quantize, quest_dequantize, alpha_of, bits, seed=0, n=6):
    """Codes in range; every unclipped element sits at its nearest level
    (brute force over all levels); clipped elements take the end codes; the
    stored delta is fp16(alpha * rms / 2^(b-1)) computed with exact sums."""
    g = np.random.default_rng(seed + bits)
    L = 1 << bits
    alpha = alpha_of(bits)
    x = g.standard_normal((n, 128)).astype(np.float32)
    x[:, :4] *= 25.0                       # outliers that clip
    x = x.astype(np.float16).astype(np.float32)
    codes, delta = quest_quantize(x, bits, alpha)
    assert codes.min() >= 0 and codes.max() < L
    xh = quest_dequantize(codes, delta, bits)
    for i in range(n):
        row = [float(v) for v in x[i]]
        rms = math.sqrt(math.fsum(v * v for v in row) / 128.0)
        want = brute.fp16_round_exact(alpha * rms / 2 ** (bits - 1))
        assert float(delta[i]) == want, (float(delta[i]), want)
        d = float(delta[i])
        lv = [(j - L / 2 + 0.5) * d for j in range(L)]
        for j, v in enumerate(row):
            c = int(codes[i, j])
            assert xh[i, j] == lv[c]
            if v >= (L / 2) * d:
                assert c == L - 1
            elif v < -(L / 2) * d:
                assert c == 0
            else:
                near = brute.nearest_level(v, lv)
                # a tie only happens on a bin edge, where floor picks the upper
                assert c in near, (v, c, near)
                assert abs(v - lv[c]) <= d / 2 * (1 + 1e-6)


def check_quest_symmetries(quest_quantize, alpha_of, bits, seed=1):
    """Doubling the input doubles delta and keeps the codes; the all-zero
    token has delta 0 and reconstructs to zero (code L/2)."""
    g = np.random.default_rng(seed)
    L = 1 << bits
    x = g.standard_normal((4, 128)).astype(np.float16).astype(np.float32)
    c1, d1 = quest_quantize(x, bits, alpha_of(bits))
    c2, d2 = quest_quantize(2 * x, bits, alpha_of(bits))
    assert (c1 == c2).all() and (d2.astype(np.float32) == 2 * d1.astype(np.float32)).all()
    cz, dz = quest_quantize(np.zeros((1, 128), np.float32), bits, alpha_of(bits))
    assert float(dz[0]) == 0.0 and (cz == L // 2).all()


def check_error_decreases_with_bits(quest_quantize, quest_dequantize, alpha_of, seed=2):
    g = np.random.default_rng(seed)
    x = g.standard_normal((64, 128)).astype(np.float16).astype(np.float32)
    errs = []
    for b in (2, 3, 4, 6, 8):
        c, d = quest_quantize(x, b, alpha_of(b))
        errs.append(np.mean((quest_dequantize(c, d, b) - x) ** 2))
    assert all(e1 > 1.5 * e2 for e1, e2 in zip(errs, errs[1:])), errs


# --- percentile-clipped affine -----------------------------------------------

def check_affine_brute(affine_quantize, affine_dequantize, bits, r_lo=2, r_hi=127, seed=3, n=6):
    """Codes in range; lo is the r_lo-th smallest value; exactly r_lo - 1
    elements fall below lo and 128 - r_hi above hi (distinct inputs); each
    element inside [lo, hi] sits at its nearest level lo + i s."""
    g = np.random.default_rng(seed + bits)
    L = 1 << bits
    x = g.standard_normal((n, 128)).astype(np.float16).astype(np.float32)
    codes, s, lo = affine_quantize(x, bits, r_lo, r_hi)
    assert codes.min() >= 0 and codes.max() < L
    xh = affine_dequantize(codes, s, lo)
    for i in range(n):
        row = [float(v) for v in x[i]]
        if len(set(row)) < 128:
            continue
        srt = sorted(row)
        assert float(lo[i]) == srt[r_lo - 1]
        hi = srt[r_hi - 1]
        assert sum(v < float(lo[i]) for v in row) == r_lo - 1
        assert sum(v > hi for v in row) == 128 - r_hi
        sv = float(s[i])
        assert sv == brute.fp16_round_exact(float(np.float32(np.float32(hi - srt[r_lo - 1]) / np.float32(L - 1))))
        lv = [float(lo[i]) + j * sv for j in range(L)]
        for j, v in enumerate(row):
            c = int(codes[i, j])
            assert abs(xh[i, j] - lv[c]) <= 1e-12 * (1 + abs(lv[c]))
            if v < float(lo[i]):
                assert c == 0
            elif v > lv[-1]:
                assert c == L - 1
            else:
                assert c in brute.nearest_level(v, lv), (v, c)


def check_affine_constant(affine_quantize, affine_dequantize, bits):
    x = np.full((1, 128), 1.25, np.float32)
    c, s, lo = affine_quantize(x, bits, 2, 127)
    assert float(s[0]) == 0.0 and (c == 0).all()
    assert (affine_dequantize(c, s, lo) == 1.25).all()


# --- windows ------------------------------------------------------------------

def check_window_counts(window_split):
    for n, chunk, ns, npk, nr in _table("window_counts.txt"):
        got = window_split(int(n), 64, 256, int(chunk))
        assert got == (int(ns), int(npk), int(nr)), (n, chunk, got)


def check_window_invariants(window_split):
    for C in (8, 16):
        prev = (0, 0, 0)
        for n in range(0, 64 + 256 + 5 * C + 3):
            ns, P, nr = window_split(n, 64, 256, C)
            assert ns + P + nr == n and P % C == 0
            if n - ns >= 256:
                assert 256 <= nr < 256 + C
            assert P >= prev[1]
            prev = (ns, P, nr)


# --- transforms and attention ------------------------------------------------

def _rand_T(g, d):
    a = g.standard_normal((d, d))
    return a + d ** 0.5 * np.eye(d)


def check_transform_invariance(transform_keys, transform_query, seed=4):
    """q'.k' = q.k when q' uses the inverse transpose of the key transform."""
    g = np.random.default_rng(seed)
    d = 128
    T = _rand_T(g, d)
    TinvT = np.linalg.inv(T).T
    k = g.standard_normal((16, d))
    q = g.standard_normal((3, d))
    lhs = transform_query(q, TinvT) @ transform_keys(k, T).T
    assert np.allclose(lhs, q @ k.T, rtol=0, atol=1e-10 * np.abs(q @ k.T).max())


def check_transform_brute(transform_keys, seed=5):
    """k' = T k matches an explicit loop on a tiny non-symmetric T."""
    g = np.random.default_rng(seed)
    T = g.standard_normal((5, 5))
    k = g.standard_normal(5)
    want = brute.matvec(T.tolist(), k.tolist())
    assert np.allclose(transform_keys(k[None], T)[0], want, rtol=1e-14, atol=1e-14)


def check_attention_brute(attention_f64, seed=6):
    g = np.random.default_rng(seed)
    for n, d in ((1, 4), (5, 8), (16, 16)):
        q = g.standard_normal(d)
        K = g.standard_normal((n, d))
        V = g.standard_normal((n, d))
        want = brute.attention_loops(q.tolist(), K.tolist(), V.tolist(), 0.3)
        got = attention_f64(q[None], K, V, 0.3)[0]
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def check_attention_through_transforms(attention_f64, transform_keys, transform_query, seed=7):
    """Unquantised attention through T and T^{-T} equals plain attention."""
    g = np.random.default_rng(seed)
    d, n = 128, 300
    T = _rand_T(g, d) / 3.0
    TinvT = np.linalg.inv(T).T
    q = g.standard_normal((4, d))
    K = g.standard_normal((n, d))
    V = g.standard_normal((n, d))
    s = 1 / math.sqrt(d)
    a = attention_f64(transform_query(q, TinvT), transform_keys(K, T), V, s)
    b = attention_f64(q, K, V, s)
    assert np.abs(a - b).max() <= 1e-12
