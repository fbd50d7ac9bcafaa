"""Chunked-prefill attention over the quantised cache: the oracle against
what fixes it (CPU), and the library against the oracle (GPU).

Reading: the chunk's n_q tokens are appended first; the query of token
p = n - n_q + i attends to tokens 0 .. p as the cache holds them (fp16 sink
and recent windows, dequantised packed tokens), as a decode query attends
after its own token was appended."""
import math

import numpy as np
import pytest

from oracle import wushkv_oracle as O
from tests import gpu_helpers as H

DECODE_TOL = 2e-3


def _filled(n, G=4, Hkv=2, B=2, bits=2, quantizer=O.QUEST_INT, sink=16, recent=32, chunk=8, seed=0,
            last_token_seed=None):
    g = np.random.default_rng(seed)
    k = g.standard_normal((B, n, Hkv, 128))
    k[..., :4] *= 12.0
    v = g.standard_normal((B, n, Hkv, 128))
    if last_token_seed is not None:
        h = np.random.default_rng(last_token_seed)
        k[:, -1] = h.standard_normal((B, Hkv, 128))
        v[:, -1] = h.standard_normal((B, Hkv, 128))
    T = np.stack([np.eye(128) + 0.2 * g.standard_normal((128, 128)) for _ in range(Hkv)])
    cfg = O.CacheConfig(B, Hkv, Hkv * G, n, bits=bits, quantizer=quantizer, sink=sink, recent=recent,
                        chunk=chunk)
    c = O.OracleCache(cfg)
    c.append(k, v, T)
    return c, k, v, T


def _oracle(c, q):
    return c.prefill_attention(q)


def check_last_query_is_the_decode(prefill):
    c, *_ = _filled(120)
    q = np.random.default_rng(1).standard_normal((2, 5, 8, 128))
    out = prefill(c, q)
    dec = c.decode(q[:, -1])
    assert np.abs(out[:, -1] - dec).max() <= 1e-12


def check_causal(prefill):
    q = np.random.default_rng(2).standard_normal((2, 6, 8, 128))
    a, *_ = _filled(130, last_token_seed=5)
    b, *_ = _filled(130, last_token_seed=6)
    oa, ob = prefill(a, q), prefill(b, q)
    assert np.array_equal(oa[:, :-1], ob[:, :-1])
    assert np.abs(oa[:, -1] - ob[:, -1]).max() > 1e-3


def test_last_query_is_the_decode():
    """The chunk's last query sees the whole cache: it is the decode of that
    query."""
    check_last_query_is_the_decode(_oracle)


def test_causal():
    """Replacing the last token changes only the last query's output."""
    check_causal(_oracle)


def _mutant(first_visible=0, extra=1, shift=0):
    """prefill_attention with a planted mistake: the query of token p sees
    tokens first_visible .. p + extra - 1 (with p moved by shift)."""
    def f(c, q):
        B, nq, Hq, d = q.shape
        G = c.cfg.group
        out = np.full((B, nq, Hq, d), np.nan)
        for u in range(c.cfg.units):
            b, h = divmod(u, c.cfg.n_kv_heads)
            K, V = c.unit_kv(u)
            for i in range(nq):
                p = c.n - nq + i + shift
                hi = min(c.n, max(p + extra, first_visible + 1))
                out[b, i, h * G:(h + 1) * G] = O.attention_f64(q[b, i, h * G:(h + 1) * G], K[first_visible:hi],
                                                               V[first_visible:hi], 1.0 / math.sqrt(128.0))
        return out
    return f


@pytest.mark.parametrize("mut", [dict(extra=0), dict(extra=10 ** 9), dict(shift=-1), dict(first_visible=1)],
                         ids=["sees-one-less", "not-causal", "position-off-by-one", "drops-token-0"])
def test_prefill_mistakes_are_caught(mut):
    """Each planted mistake fails at least one pin."""
    bad = _mutant(**mut)
    caught = 0
    for check in (check_last_query_is_the_decode, check_causal, check_brute_force_tiny):
        try:
            check(bad)
        except AssertionError:
            caught += 1
    assert caught >= 1, mut


def test_brute_force_tiny():
    """Explicit loops over tokens (max, exponentials, sums) on a tiny cache
    with sink, packed and recent tokens."""
    check_brute_force_tiny(_oracle)


def check_brute_force_tiny(prefill):
    c, *_ = _filled(45, G=2, Hkv=1, B=1, sink=4, recent=8, chunk=4, seed=3)
    assert c.split()[1] > 0
    q = np.random.default_rng(4).standard_normal((1, 7, 2, 128))
    out = prefill(c, q)
    K, V = c.unit_kv(0)
    s = 1.0 / math.sqrt(128.0)
    for i in range(7):
        p = 45 - 7 + i
        for hh in range(2):
            scores = [s * sum(q[0, i, hh, d] * K[t, d] for d in range(128)) for t in range(p + 1)]
            m = max(scores)
            w = [math.exp(x - m) for x in scores]
            z = sum(w)
            ref = [sum(w[t] * V[t, d] for t in range(p + 1)) / z for d in range(128)]
            assert np.abs(out[0, i, hh] - np.array(ref)).max() <= 1e-12


def test_windows_only_is_causal_attention():
    """Nothing packed: the chunk's outputs are causal softmax attention over
    the fp16-rounded transformed keys and fp16 values, one masked matrix
    product per head."""
    n, G = 60, 4
    c, k, v, T = _filled(n, G=G, recent=256, sink=16)
    assert c.split()[1] == 0
    nq = 20
    q = np.random.default_rng(7).standard_normal((2, nq, 2 * G, 128))
    out = c.prefill_attention(q)
    s = 1.0 / math.sqrt(128.0)
    pos = np.arange(n - nq, n)
    mask = np.arange(n)[None, :] > pos[:, None]
    for b in range(2):
        for h in range(2 * G):
            kv = h // G
            K = (k[b, :, kv] @ T[kv].T).astype(np.float16).astype(np.float64)
            Vv = v[b, :, kv].astype(np.float16).astype(np.float64)
            S = s * q[b, :, h] @ K.T
            S[mask] = -np.inf
            P = np.exp(S - S.max(axis=1, keepdims=True))
            ref = (P / P.sum(axis=1, keepdims=True)) @ Vv
            assert np.abs(out[b, :, h] - ref).max() <= 1e-12


# ---------------------------------------------------------------------------
# The library against the oracle (needs a B200)
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def wk():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_post_b200 import wushkv
    wushkv.load()
    return wushkv


def _gpu_case(wk, n, nq, G, bits, quantizer, B=2, Hkv=2, seed=0, paged=False):
    """The same transformed fp16 keys and values into both caches (keys
    passed with no transform, so both caches are bit-identical), then the
    chunk's queries through both prefill attentions."""
    import torch
    g = np.random.default_rng(seed)
    kt = g.standard_normal((B, n, Hkv, 128)).astype(np.float32)
    kt[..., :8] *= 10.0
    vt = g.standard_normal((B, n, Hkv, 128)).astype(np.float32)
    kt, vt = H.rounded(kt, "f16"), H.rounded(vt, "f16")
    cfg = wk.make_config(B, Hkv, Hkv * G, n + 64, bits=bits, quantizer=quantizer,
                         num_pages=(B * ((n + 64 + 127) // 128 * 2) + 3) if paged else 0)
    cache = wk.Cache(cfg)
    if paged:
        per = (cfg.max_ctx + 127) // 128 * 2
        perm = np.random.default_rng(seed + 1).permutation(cfg.num_pages)[:B * per].reshape(B, per)
        cache.set_page_table(torch.from_numpy(perm.astype(np.int32)).cuda(), per)
    cache.append(H.to_dev(kt, "f16"), H.to_dev(vt, "f16"), None)
    oc = O.OracleCache(H.oracle_cfg(cfg))
    oc.append(kt.astype(np.float64), vt.astype(np.float64), None)
    q = g.standard_normal((B, nq, Hkv * G, 128)).astype(np.float32)
    out = cache.prefill_attention(torch.from_numpy(q).cuda(), nq).cpu().numpy()
    assert cache.device_status() == 0
    H.check_guards(cache)
    return out, oc.prefill_attention(q.astype(np.float64)), cache, oc, q


@pytest.mark.gpu
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("quantizer", [0, 1])
def test_prefill_attention_matches_oracle(wk, bits, quantizer):
    out, ref, *_ = _gpu_case(wk, 700, 150, 4, bits, quantizer)
    err = np.abs(out - ref).max() / math.sqrt(float(np.mean(ref ** 2)))
    assert err <= DECODE_TOL, err


@pytest.mark.gpu
@pytest.mark.parametrize("G", [1, 2, 8])
def test_prefill_attention_groups(wk, G):
    out, ref, *_ = _gpu_case(wk, 420, 37, G, 2, 0, seed=G)
    err = np.abs(out - ref).max() / math.sqrt(float(np.mean(ref ** 2)))
    assert err <= DECODE_TOL, err


@pytest.mark.gpu
@pytest.mark.parametrize("n,nq", [(9, 9), (64, 1), (330, 330), (1000, 64)])
def test_prefill_attention_edges(wk, n, nq):
    """Whole-cache chunks (every token a query), a one-token chunk, chunks
    that end inside the sink, the packed region and the ring."""
    out, ref, *_ = _gpu_case(wk, n, nq, 4, 2, 0, seed=n)
    err = np.abs(out - ref).max() / math.sqrt(float(np.mean(ref ** 2)))
    assert err <= DECODE_TOL, err


@pytest.mark.gpu
def test_prefill_attention_paged(wk):
    out, ref, *_ = _gpu_case(wk, 900, 80, 4, 2, 1, seed=11, paged=True)
    err = np.abs(out - ref).max() / math.sqrt(float(np.mean(ref ** 2)))
    assert err <= DECODE_TOL, err


@pytest.mark.gpu
def test_prefill_attention_last_row_is_decode(wk):
    """The chunk's last query against the library's own decode."""
    import torch
    out, ref, cache, oc, q = _gpu_case(wk, 600, 40, 4, 2, 0, seed=21)
    dec = cache.decode(torch.from_numpy(np.ascontiguousarray(q[:, -1])).cuda()).cpu().numpy()
    rms = math.sqrt(float(np.mean(dec.astype(np.float64) ** 2)))
    assert np.abs(out[:, -1] - dec).max() / rms <= DECODE_TOL


@pytest.mark.gpu
def test_prefill_attention_qwen3_8b_layer_chunk512(wk):
    """Full-size Qwen3-8B-shaped layer (batch 16, 8 KV heads, G 4, bf16):
    8192 tokens appended through the key transform, the last 512 of them
    the chunk.  Sampled units and queries against float64 causal attention
    over the GPU cache's own state (read through wushkv_export and
    dequantised with the oracle's rules)."""
    import torch
    from bit_kv_cache_post_b200 import inputs as I
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    n, nq, G = w.context, 512, w.group
    k, v = I.device_kv(w, 0, n)
    T, TinvT = I.key_transforms(w, 0)
    cache = wk.Cache(wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, n, bits=2))
    cache.append(k, v, torch.from_numpy(T).cuda())
    del k, v
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    q = torch.randn((w.batch * nq, w.n_q_heads, 128), generator=g, device="cuda").bfloat16()
    qp = wk.query_transform(q, torch.from_numpy(TinvT).cuda()).view(w.batch, nq, w.n_q_heads, 128)
    out = cache.prefill_attention(qp.contiguous(), nq).cpu().numpy()
    qp = qp.cpu().numpy().astype(np.float64)
    assert cache.device_status() == 0
    rng = np.random.default_rng(5)
    for b, h in [(0, 0), (15, 7), (int(rng.integers(16)), int(rng.integers(8)))]:
        Kg, Vg = H.unit_state_from_export(cache, b, h)
        for i in sorted(set([0, nq - 1] + list(rng.integers(0, nq, 6)))):
            p = n - nq + i
            want = O.attention_f64(qp[b, i, h * G:(h + 1) * G], Kg[:p + 1], Vg[:p + 1], 1.0 / np.sqrt(128.0))
            got = out[b, i, h * G:(h + 1) * G]
            assert np.abs(got - want).max() / math.sqrt(float(np.mean(want ** 2))) <= DECODE_TOL, (b, h, i)
    H.check_guards(cache)
