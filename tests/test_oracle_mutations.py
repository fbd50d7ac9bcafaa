"""Each pin must catch a plausible mistake planted in a copy of the oracle.

The mistakes are planted here, on the CPU, in wrapped copies of the oracle's
functions; the oracle itself is untouched.
"""
import math

import numpy as np
import pytest

from oracle import wushkv_oracle as O
from tests import oracle_pins as P


def _fails(check, *args, **kw):
    with pytest.raises(AssertionError):
        check(*args, **kw)


def test_transposed_key_transform_is_caught():
    bad = lambda k, T: np.asarray(k, np.float64) @ np.asarray(T, np.float64)
    _fails(P.check_transform_brute, bad)
    _fails(P.check_transform_invariance, bad, O.transform_query)


def test_query_transform_without_inverse_is_caught():
    bad = lambda q, TinvT: np.asarray(q, np.float64) @ np.linalg.inv(np.asarray(TinvT, np.float64).T).T
    _fails(P.check_transform_invariance, O.transform_keys, bad)


def test_missing_attention_scale_is_caught():
    bad = lambda q, K, V, s: O.attention_f64(q, K, V, 1.0)
    _fails(P.check_attention_brute, bad)


def test_softmax_over_wrong_axis_is_caught():
    def bad(q, K, V, scale):
        s = scale * (np.atleast_2d(q) @ K.T)
        p = np.exp(s - s.max(axis=0, keepdims=True))
        return (p / p.sum(axis=0, keepdims=True)) @ V
    _fails(P.check_attention_brute, bad)


def _quest_variant(rms_div=True, centre=0.5, use_rint=False, pow_off=1):
    def q(x, bits, alpha):
        x32 = np.asarray(x, np.float32)
        L = 1 << bits
        ss = np.sum(x32.astype(np.float64) ** 2, axis=-1)
        rms = np.sqrt(ss / 128.0) if rms_div else np.sqrt(ss)
        d = (alpha * rms / float(1 << (bits - pow_off))).astype(np.float16)
        d32 = d.astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            t = (x32 * (np.float32(1) / d32)[..., None]).astype(np.float32) + np.float32(L // 2)
        t = np.where((d32 == 0)[..., None], np.float32(L // 2), t)
        r = np.rint(t) if use_rint else np.floor(t)
        return np.clip(r, 0, L - 1).astype(np.uint8), d

    def dq(codes, d, bits):
        L = 1 << bits
        return (codes.astype(np.float64) - L / 2 + centre) * d.astype(np.float64)[..., None]
    return q, dq


@pytest.mark.parametrize("variant", [dict(rms_div=False), dict(centre=0.0), dict(use_rint=True),
                                     dict(pow_off=0)])
def test_quest_mistakes_are_caught(variant):
    q, dq = _quest_variant(**variant)
    _fails(P.check_quest_brute, q, dq, O.quest_alpha, 2)


def test_wrong_clip_ratio_is_caught():
    _fails(P.check_alpha_max_table, lambda b: 1.1 * O.quest_alpha(b), O.uniform_gaussian_mse)
    _fails(P.check_alpha_max_table, lambda b: O.quest_alpha(b + 1), O.uniform_gaussian_mse)


def test_affine_rank_off_by_one_is_caught():
    def bad(x, bits, r_lo, r_hi):
        return O.affine_quantize(x, bits, r_lo + 1, r_hi)
    _fails(P.check_affine_brute, bad, O.affine_dequantize, 2)


def test_affine_missing_offset_is_caught():
    bad_dq = lambda c, s, lo: c.astype(np.float64) * s.astype(np.float64)[..., None]
    _fails(P.check_affine_brute, O.affine_quantize, bad_dq, 2)


def test_affine_floor_instead_of_round_is_caught():
    def bad(x, bits, r_lo, r_hi):
        x32 = np.asarray(x, np.float32)
        L = 1 << bits
        srt = np.sort(x32, axis=-1)
        lo, hi = srt[..., r_lo - 1], srt[..., r_hi - 1]
        s = ((hi - lo) / np.float32(L - 1)).astype(np.float16)
        t = (x32 - lo.astype(np.float16).astype(np.float32)[..., None]) / s.astype(np.float32)[..., None]
        return np.clip(np.floor(t), 0, L - 1).astype(np.uint8), s, lo.astype(np.float16)
    _fails(P.check_affine_brute, bad, O.affine_dequantize, 2)


def test_flush_threshold_mistakes_are_caught():
    def flush_at_recent(n, sink, recent, chunk):
        ns = min(n, sink)
        m = n - ns
        packed = chunk * ((m - recent + chunk) // chunk) if m >= recent else 0
        return ns, packed, m - packed
    _fails(P.check_window_counts, flush_at_recent)

    def no_sink(n, sink, recent, chunk):
        packed = chunk * ((n - recent) // chunk) if n >= recent + chunk else 0
        return 0, packed, n - packed
    _fails(P.check_window_counts, no_sink)


def test_gqa_grouping_pin():
    """Head h reads KV head h // G: with T^{-T} = I for KV head 0 and 2 I for
    KV head 1, the first G query heads pass through and the rest double."""
    G = 4
    q = np.random.default_rng(0).standard_normal((1, 2 * G, 128))
    TinvT = np.stack([np.eye(128), 2 * np.eye(128)])

    def check(fn):
        out = fn(q, TinvT)
        assert np.array_equal(out[0, :G], q[0, :G]) and np.array_equal(out[0, G:], 2 * q[0, G:])

    check(O.query_transform_gqa)

    def interleaved(qq, T):
        out = np.empty_like(qq)
        for h in range(qq.shape[1]):
            out[:, h] = qq[:, h] @ T[h % T.shape[0]].T
        return out
    _fails(check, interleaved)
