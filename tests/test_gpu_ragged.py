"""Sequences of different lengths and the paged packed region against the
CPU oracle (needs a B200).

Each sequence of a ragged batch is its own batch-1 oracle cache: the window
policy (sink, recent ring, chunked flush) applies to every sequence on its
own, so the oracle needs no new arithmetic.  Caches are compared through
wushkv_export (which reads pages through the page table) and decodes within
the decode tolerance."""
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


def _tokens(seed, n, Hkv):
    g = np.random.default_rng(seed)
    k = g.standard_normal((n, Hkv, 128)).astype(np.float32)
    k[:, :, g.choice(128, 8, replace=False)] *= 20.0
    v = g.standard_normal((n, Hkv, 128)).astype(np.float32)
    return k, v


def _paged(wk, cfg, B, seed):
    """A page table giving every sequence a random set of distinct pages."""
    import torch
    cap_blocks = (cfg.max_ctx + 127) // 128 * 2
    perm = np.random.default_rng(seed).permutation(cfg.num_pages)[:B * cap_blocks].reshape(B, cap_blocks)
    return torch.from_numpy(perm.astype(np.int32)).cuda(), cap_blocks


def _run_schedule(wk, cache, ocs, schedule, Hkv, dtype, T, seed):
    """schedule: list of per-sequence new-token counts, one entry per call."""
    import torch
    Td = None if T is None else torch.from_numpy(T).cuda()
    for step, counts in enumerate(schedule):
        ks, vs = [], []
        for b, c in enumerate(counts):
            k, v = _tokens(seed * 1000 + step * 37 + b, c, Hkv)
            k, v = H.rounded(k, dtype), H.rounded(v, dtype)
            ks.append(k)
            vs.append(v)
            if c:
                ocs[b].append(k[None], v[None], None if T is None else T.astype(np.float64))
        k = np.concatenate(ks) if sum(counts) else np.zeros((0, Hkv, 128), np.float32)
        v = np.concatenate(vs) if sum(counts) else np.zeros((0, Hkv, 128), np.float32)
        if sum(counts):
            cache.append_varlen(H.to_dev(k, dtype), H.to_dev(v, dtype), counts, Td)
    torch.cuda.synchronize()
    assert cache.device_status() == 0


def _decode_check(wk, cache, ocs, B, Hkv, G, seed):
    import torch
    q = np.random.default_rng(seed).standard_normal((B, Hkv * G, 128)).astype(np.float32)
    out = torch.full((B, Hkv * G, 128), float("nan"), device="cuda")
    cache.decode(torch.from_numpy(q).cuda(), out=out)
    out = out.cpu().numpy()
    for b in range(B):
        if ocs[b].n == 0:
            assert np.isnan(out[b]).all()        # rows of an empty sequence are left unchanged
            continue
        want = ocs[b].decode(q[b:b + 1].astype(np.float64))[0]
        assert H.rel_rms_err(out[b], want) <= DECODE_TOL, b
    assert cache.device_status() == 0
    return out


RAGGED = [[700, 9, 0, 331], [1, 1, 0, 1], [300, 0, 400, 8], [1, 1, 1, 0], [0, 250, 5, 1]]


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("bits,quantizer", [(2, O.QUEST_INT), (3, O.AFFINE_PCTCLIP), (4, O.QUEST_INT)])
def test_ragged_cache_bitexact_and_decode(wk, bits, quantizer, paged):
    """Appends of different sizes per sequence (including none), bulk and
    single-token, on dense and paged caches: every unit's stored state is the
    oracle's, and one decode serves all sequences at their own lengths."""
    import torch
    B, Hkv, G = 4, 2, 4
    cfg = wk.make_config(B, Hkv, Hkv * G, 1100, bits=bits, quantizer=quantizer,
                         num_pages=(B * 18 + 7) if paged else 0)
    cache = wk.Cache(cfg)
    if paged:
        pt, stride = _paged(wk, cfg, B, bits)
        cache.set_page_table(pt, stride)
    ocs = [O.OracleCache(O.CacheConfig(1, Hkv, Hkv * G, 1100, bits=bits, quantizer=quantizer)) for _ in range(B)]
    _run_schedule(wk, cache, ocs, RAGGED, Hkv, "f32", None, bits)
    for b in range(B):
        assert cache.tokens(b)[0] == ocs[b].n
        for h in range(Hkv):
            H.compare_unit_by_export(cache, b, h, ocs[b], h)
    _decode_check(wk, cache, ocs, B, Hkv, G, 3)
    H.check_guards(cache)


@pytest.mark.parametrize("paged", [False, True])
def test_ragged_bf16_through_transform(wk, paged):
    """bf16 keys through T with per-sequence bulk prefills (the tensor-core
    path runs per sequence) then single-token steps; keys within the
    transform tolerances of the oracle's, decode within tolerance."""
    import torch
    B, Hkv, G = 3, 2, 4
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    T, TinvT = I.key_transforms(w, 2)
    T, TinvT = T[:Hkv], TinvT[:Hkv]
    cfg = wk.make_config(B, Hkv, Hkv * G, 1400, bits=2, num_pages=(B * 22 + 3) if paged else 0)
    cache = wk.Cache(cfg)
    if paged:
        pt, stride = _paged(wk, cfg, B, 9)
        cache.set_page_table(pt, stride)
    ocs = [O.OracleCache(O.CacheConfig(1, Hkv, Hkv * G, 1400, bits=2)) for _ in range(B)]
    sched = [[900, 300, 1200]] + [[1, 1, 1]] * 9
    _run_schedule(wk, cache, ocs, sched, Hkv, "bf16", T, 5)
    q = np.random.default_rng(1).standard_normal((B, Hkv * G, 128)).astype(np.float32)
    qp = wk.query_transform(torch.from_numpy(q).cuda(), torch.from_numpy(TinvT).cuda())
    out = cache.decode(qp).cpu().numpy()
    for b in range(B):
        ns, P, nr = ocs[b].split()
        n = ocs[b].n
        for h in range(Hkv):
            codes, _, rows, kinds = cache.export(b, h, 0, 0, n)
            assert np.array_equal(kinds, np.array([0] * ns + [1] * P + [2] * nr, np.int8))
            if P:
                mism = float(np.mean(codes[ns:ns + P] != ocs[b].codes_k[h, :P]))
                assert mism <= 1e-4, (b, h, mism)
        # decode against exact attention over the state the GPU built
        for h in range(Hkv):
            Kg, Vg = H.unit_state_from_export(cache, b, h)
            qpr = O.transform_query(q[b, h * G:(h + 1) * G], TinvT[h].astype(np.float64))
            want = O.attention_f64(qpr, Kg, Vg, 1.0 / np.sqrt(128.0))
            assert H.rel_rms_err(out[b, h * G:(h + 1) * G], want) <= DECODE_TOL
    assert cache.device_status() == 0
    H.check_guards(cache)


def test_reset_sequence_and_refill(wk):
    """A sequence emptied and refilled (a new request in its batch slot)
    holds only the new tokens; the other sequences are untouched."""
    B, Hkv, G = 3, 2, 2
    cfg = wk.make_config(B, Hkv, Hkv * G, 900, bits=2)
    cache = wk.Cache(cfg)
    ocs = [O.OracleCache(O.CacheConfig(1, Hkv, Hkv * G, 900, bits=2)) for _ in range(B)]
    _run_schedule(wk, cache, ocs, [[500, 400, 600]], Hkv, "f32", None, 1)
    cache.reset_sequence(1)
    assert cache.tokens(1) == (0, 0, 0, 0)
    ocs[1] = O.OracleCache(O.CacheConfig(1, Hkv, Hkv * G, 900, bits=2))
    _decode_check(wk, cache, ocs, B, Hkv, G, 6)          # sequence 1 empty: its rows untouched
    _run_schedule(wk, cache, ocs, [[0, 350, 0], [1, 1, 1]], Hkv, "f32", None, 2)
    for b in range(B):
        for h in range(Hkv):
            H.compare_unit_by_export(cache, b, h, ocs[b], h)
    _decode_check(wk, cache, ocs, B, Hkv, G, 4)


def test_ragged_decode_step_equals_separate_calls(wk):
    """On a ragged cache the one-call step is the per-sequence append, the
    query transform and the ragged decode: identical results."""
    import torch
    B, Hkv, G = 3, 2, 4
    w = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]
    T, TinvT = I.key_transforms(w, 4)
    Td, TiTd = torch.from_numpy(T[:Hkv]).cuda(), torch.from_numpy(TinvT[:Hkv]).cuda()
    cfg = wk.make_config(B, Hkv, Hkv * G, 800, bits=2)
    a, b_ = wk.Cache(cfg), wk.Cache(cfg)
    k0, v0 = _tokens(1, 1500, Hkv)
    for c in (a, b_):
        c.append_varlen(H.to_dev(k0, "bf16"), H.to_dev(v0, "bf16"), [700, 300, 500], Td)
    for s in range(12):
        k, v = _tokens(100 + s, B, Hkv)
        kd, vd = H.to_dev(k[:, None], "bf16"), H.to_dev(v[:, None], "bf16")
        q = H.to_dev(np.random.default_rng(s).standard_normal((B, Hkv * G, 128)), "bf16")
        qa = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        out_a = a.decode_step(kd, vd, Td, q, TiTd, q_prime=qa)
        b_.append(kd, vd, Td)
        out_b = b_.decode(wk.query_transform(q, TiTd))
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b), s
    assert [a.tokens(x)[0] for x in range(B)] == [712, 312, 512]
