"""The CPU oracle against its pins (no GPU)."""
import math

import numpy as np
import pytest

from oracle import brute
from oracle import wushkv_oracle as O
from tests import oracle_pins as P


def test_alpha_matches_max_table():
    P.check_alpha_max_table(O.quest_alpha, O.uniform_gaussian_mse)


def test_alpha_is_a_minimum():
    for b in (2, 3, 4):
        a, L = O.quest_alpha(b), 1 << b
        f = O.uniform_gaussian_mse
        assert f(a, L) < f(a * 1.001, L) and f(a, L) < f(a * 0.999, L)
        assert abs(O.uniform_gaussian_mse_deriv(a, L)) < 1e-12


def test_mse_monte_carlo():
    P.check_mse_monte_carlo(O.uniform_gaussian_mse)


def test_fp16_rounding_primitive():
    """numpy's float64 -> fp16 conversion (used by the oracle for the stored
    scales and transformed keys) rounds once, to nearest even."""
    g = np.random.default_rng(0)
    xs = np.concatenate([g.standard_normal(300) * 10.0 ** g.integers(-6, 4, 300),
                         [1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -24 * 1.5, 65519.9, 1 + 2 ** -11 + 2 ** -40]])
    for x in xs:
        assert float(np.float16(np.float64(x))) == brute.fp16_round_exact(float(x)), x


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quest_brute_force(bits):
    P.check_quest_brute(O.quest_quantize, O.quest_dequantize, O.quest_alpha, bits)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quest_symmetries(bits):
    P.check_quest_symmetries(O.quest_quantize, O.quest_alpha, bits)


def test_quest_error_decreases_with_bits():
    P.check_error_decreases_with_bits(O.quest_quantize, O.quest_dequantize, O.quest_alpha)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_affine_brute_force(bits):
    P.check_affine_brute(O.affine_quantize, O.affine_dequantize, bits)
    P.check_affine_brute(O.affine_quantize, O.affine_dequantize, bits, r_lo=1, r_hi=128, seed=9)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_affine_constant_token(bits):
    P.check_affine_constant(O.affine_quantize, O.affine_dequantize, bits)


def test_window_counts():
    P.check_window_counts(O.window_split)


def test_window_invariants():
    P.check_window_invariants(O.window_split)


def test_transform_invariance():
    P.check_transform_invariance(O.transform_keys, O.transform_query)


def test_transform_brute():
    P.check_transform_brute(O.transform_keys)


def test_attention_brute():
    P.check_attention_brute(O.attention_f64)


def test_attention_through_transforms():
    P.check_attention_through_transforms(O.attention_f64, O.transform_keys, O.transform_query)


# --- packed byte format -------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip_and_bijection(bits):
    g = np.random.default_rng(bits)
    c = g.integers(0, 1 << bits, (8, 128)).astype(np.uint8)
    assert (O.unpack_k_rows(O.pack_k_rows(c, bits), bits) == c).all()
    cq = g.integers(0, 1 << bits, (3, 4, 128)).astype(np.uint8)
    assert (O.unpack_v_quads(O.pack_v_quads(cq, bits), bits) == cq).all()
    # every (dim) of a row and every (token, dim) of a quad owns distinct bits
    total = sum(int(np.unpackbits(p.view(np.uint8)).sum())
                for p in O.pack_k_rows(np.full((4, 128), (1 << bits) - 1, np.uint8), bits))
    assert total == 4 * 128 * bits
    total = sum(int(np.unpackbits(p.view(np.uint8)).sum())
                for p in O.pack_v_quads(np.full((1, 4, 128), (1 << bits) - 1, np.uint8), bits))
    assert total == 512 * bits


def _golden_positions():
    rows = []
    for line in open(P.GOLDEN + "/pack_positions.txt"):
        line = line.split("#", 1)[0].strip()
        if line:
            kind, bits, plane, tok, dim, word, bit = line.split()
            rows.append((kind, int(bits), int(plane), int(tok), int(dim), int(word), int(bit)))
    return rows


def test_pack_positions_golden():
    """A single code at one (token, dim) lands on the hand-derived word and
    bit of the documented format."""
    for kind, bits, plane, tok, dim, word, bit in _golden_positions():
        code = (1 << bits) - 1
        if kind == "K":
            c = np.zeros(((tok // 4 + 1) * 4 if bits == 2 else 1, 128), np.uint8)
            c[tok if bits == 2 else 0, dim] = code
            planes = O.pack_k_rows(c, bits)
        else:
            c = np.zeros((tok // 4 + 1, 4, 128), np.uint8)
            c[tok // 4, tok % 4, dim] = code
            planes = O.pack_v_quads(c, bits)
        words = planes[plane].reshape(-1)
        nz = np.flatnonzero(words)
        assert list(nz) == [word], (kind, bits, dim, nz)
        assert (int(words[word]) >> bit) & 1 == 1 and int(words[word]) & ((1 << bit) - 1) == 0


# --- cache-level pins -----------------------------------------------------------

def _cache(n, chunk=8, bits=2, quantizer=O.QUEST_INT, recent=256, sink=64, Hq=4,
           r_lo=2, r_hi=127):
    return O.OracleCache(O.CacheConfig(batch=2, n_kv_heads=2, n_q_heads=Hq, max_ctx=n,
                                       bits=bits, quantizer=quantizer, sink=sink,
                                       recent=recent, chunk=chunk, r_lo=r_lo, r_hi=r_hi))


def test_bulk_equals_token_by_token():
    g = np.random.default_rng(11)
    n = 420
    k = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    v = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    T = np.stack([np.eye(128) + 0.1 * g.standard_normal((128, 128)) for _ in range(2)])
    a, b = _cache(n), _cache(n)
    a.append(k, v, T)
    i = 0
    for step in (1, 7, 64, 3, 200, 1, 1, 143):
        b.append(k[:, i:i + step], v[:, i:i + step], T)
        i += step
    assert i == n
    for name in ("sink_k", "sink_v", "ring_k", "ring_v", "codes_k", "codes_v", "meta_k", "meta_v"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    assert a.split() == b.split() == O.window_split(n, 64, 256, 8)


def test_windows_hold_fp16_bit_identical():
    g = np.random.default_rng(12)
    n = 400
    k = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    v = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    c = _cache(n)
    c.append(k, v, None)
    ns, P_, nr = c.split()
    order = c.recent_order()
    ku = k.transpose(0, 2, 1, 3).reshape(4, n, 128).astype(np.float16)
    vu = v.transpose(0, 2, 1, 3).reshape(4, n, 128).astype(np.float16)
    assert np.array_equal(c.sink_k[:, :ns].view(np.uint16), ku[:, :ns].view(np.uint16))
    assert np.array_equal(c.ring_k[:, order].view(np.uint16), ku[:, ns + P_:].view(np.uint16))
    assert np.array_equal(c.ring_v[:, order].view(np.uint16), vu[:, ns + P_:].view(np.uint16))


def test_decode_without_packing_is_plain_attention():
    """Nothing packed (large recent window): decode equals float64 attention
    over the fp16-rounded transformed keys, head group by head group."""
    g = np.random.default_rng(13)
    n, G = 150, 4
    k = g.standard_normal((2, n, 2, 128))
    v = g.standard_normal((2, n, 2, 128))
    T = np.stack([np.eye(128) + 0.2 * g.standard_normal((128, 128)) for _ in range(2)])
    c = _cache(n, recent=512, Hq=2 * G)
    c.append(k, v, T)
    q = g.standard_normal((2, 2 * G, 128))
    out = c.decode(q)
    s = 1 / math.sqrt(128)
    for b in range(2):
        for h in range(2 * G):
            kv = h // G
            K = (k[b, :, kv] @ T[kv].T).astype(np.float16).astype(np.float64)
            V = v[b, :, kv].astype(np.float16).astype(np.float64)
            ref = O.attention_f64(q[b, h][None], K, V, s)[0]
            assert np.abs(out[b, h] - ref).max() <= 1e-12


@pytest.mark.parametrize("quantizer", [O.QUEST_INT, O.AFFINE_PCTCLIP])
def test_decode_error_shrinks_with_bits(quantizer):
    """Quantised attention approaches unquantised attention as bits grow.
    (The affine quantiser runs unclipped, ranks 1 and 128, here: its clipped
    elements would otherwise set an error floor that bits cannot lower.)"""
    g = np.random.default_rng(14)
    n = 64 + 8 * 40 + 100
    k = g.standard_normal((2, n, 2, 128))
    v = g.standard_normal((2, n, 2, 128))
    q = g.standard_normal((2, 4, 128)) * 2.0
    T = np.stack([np.eye(128)] * 2)
    ref = _cache(n, recent=n, bits=2)
    ref.append(k, v, T)
    exact = ref.decode(q)
    errs = []
    for bits in (2, 3, 4, 6, 8):
        c = _cache(n, bits=bits, quantizer=quantizer, recent=16, sink=4, r_lo=1, r_hi=128)
        c.append(k, v, T)
        errs.append(np.sqrt(np.mean((c.decode(q) - exact) ** 2)))
    assert all(e1 > 1.4 * e2 for e1, e2 in zip(errs, errs[1:])), errs
    assert errs[-1] < 0.02 * np.sqrt(np.mean(exact ** 2))
