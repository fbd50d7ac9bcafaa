"""Host-side pieces of bench.py that need no GPU: the ragged length recipe
and the algorithmic byte and flop models."""
import numpy as np

import bench
from bit_kv_cache_post_b200 import inputs as I
from oracle import wushkv_oracle as O

W = I.WORKLOADS[bench.WORKLOAD]


def test_ragged_lengths_keep_the_total_and_spread():
    lens = bench.ragged_lengths(W)
    assert len(lens) == W.batch
    assert sum(lens) == W.batch * W.context
    assert min(lens) >= W.context // 2 and max(lens) <= W.context + W.context // 2
    assert len(set(lens)) > W.batch // 2
    assert lens == bench.ragged_lengths(W)            # seeded


def test_window_state_matches_the_oracle_split():
    for n in (1, 63, 64, 65, 320, 327, 328, 8191, 8192, 8200):
        oc_cfg = O.CacheConfig(1, 1, 4, n, sink=W.sink, recent=W.recent, chunk=W.chunk)
        assert bench.window_state(n, W)[1:] == O.window_split(n, oc_cfg.sink, oc_cfg.recent, oc_cfg.chunk)


def test_decode_bytes_count_codes_scales_and_windows():
    n, ns, P, nr = bench.window_state(8192, W)
    per_unit = P * 2 * (16 * 2 + 2) + (ns + nr) * 512
    assert bench.decode_bytes(W, 2, (n, ns, P, nr)) == W.units * per_unit + 2 * W.batch * W.n_q_heads * 512


def test_prefill_attention_flop_model():
    """4 x 128 flop per (query head, visible token), counted token by token."""
    for n, nq in ((100, 7), (8192, 512), (9, 9)):
        pairs = sum(1 for i in range(nq) for t in range(n) if t <= n - nq + i)
        assert bench.prefill_attention_flops(n, nq, 3, 5) == 4.0 * 128 * pairs * 15
