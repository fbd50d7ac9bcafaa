#!/usr/bin/env python
"""Decode-step benchmark of the WUSH-KV cache path on B200.

One step = one decode step of one Qwen3-8B-shaped layer (32 query heads, 8 KV
heads, head_dim 128, batch 16, ~8192 cached tokens, bf16 inputs, 2-bit QuEST
INT, sink 64, recent 256, chunk 8):

  append 1 post-RoPE token per sequence (key transform, fp16 recent window,
  chunked flush with quantise + pack)  ->  query transform q' = T^{-T} q
  ->  GQA decode attention over the packed cache + fp16 windows.

The timed region cycles through `--copies` independent caches (one per
"layer"), so each step reads cache bytes that are not in the 126 MB L2.

    python bench.py [--steps K] [--warmup W] [--bits 2] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N   (independent replicas)
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "qwen3-8b-layer-b16-ctx8192"
STEP_POOL = 32          # distinct per-step inputs, cycled


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--copies", type=int, default=64)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--only-prefill", action="store_true",
                    help="run only the bulk-prefill measurement (for profiling)")
    ap.add_argument("--prefill-batch", type=int, default=0,
                    help="sequences of the bulk prefill (default: the workload's 64)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# byte model: algorithmic bytes (packed codes, per-token scales, fp16 windows)
# ---------------------------------------------------------------------------

def meta_bytes(quantizer: str) -> int:
    return 2 if quantizer == "quest" else 4


def decode_bytes(w, bits, state) -> int:
    """KV bytes one decode reads (packed codes + per-token scales + fp16
    windows) plus q' read and output write."""
    _, ns, P, nr = state
    per_unit = P * 2 * (16 * bits + meta_bytes(w.quantizer)) + (ns + nr) * 2 * 256
    return w.units * per_unit + 2 * w.batch * w.n_q_heads * 128 * 4


def append_bytes(w, bits, flushed: bool) -> int:
    b = 2 * w.units * 128 * 2                 # bf16 k, v in
    b += w.n_kv_heads * 128 * 128 * 4         # T_k
    b += 2 * w.units * 128 * 2                # fp16 ring rows out
    if flushed:
        b += w.chunk * w.units * 2 * 256 + w.chunk * w.units * 2 * (16 * bits + meta_bytes(w.quantizer))
    return b


def qtransform_bytes(w) -> int:
    return w.batch * w.n_q_heads * 128 * (2 + 4) + w.n_kv_heads * 128 * 128 * 4


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (every rank gets it).  The job's
    time is the slowest rank's: each rank runs an independent replica of the
    workload (weak scaling, no data-path collective)."""
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(step_bytes_per_rank: float, ms: float, world: int) -> float:
    """Whole-job GB/s: every rank moved step_bytes_per_rank in the timed
    region, and the region took ms (max over ranks)."""
    return world * step_bytes_per_rank / (ms / 1e3) / 1e9


def build_inputs(w, torch, device):
    """Prefill keys/values (context - 1 tokens) and a pool of per-step tokens."""
    from bit_kv_cache_post_b200 import inputs as I
    n = w.context - 1
    k = np.stack([I.keys(w, 0, b, n) for b in range(w.batch)])       # [B, n, Hkv, 128]
    v = np.stack([I.values(w, 0, b, n) for b in range(w.batch)])
    kd = torch.from_numpy(k).to(device).to(torch.bfloat16)
    vd = torch.from_numpy(v).to(device).to(torch.bfloat16)
    del k, v
    pool = []
    for s in range(STEP_POOL):
        ks, vs, qs = zip(*[I.step_tokens(w, 0, b, s) for b in range(w.batch)])
        pool.append(tuple(torch.from_numpy(np.stack(x)).to(torch.bfloat16).pin_memory()
                          for x in (ks, vs, qs)))          # [B,1,Hkv,128], [B,1,Hkv,128], [B,Hq,128]
    return kd, vd, pool


def window_state(n, w):
    """(n, sink, packed, recent) token counts of one sequence (the byte model
    follows the cache's window bookkeeping)."""
    ns = min(n, w.sink)
    m = n - ns
    P = w.chunk * ((m - w.recent) // w.chunk) if m >= w.recent + w.chunk else 0
    return n, ns, P, m - P


def decode_graph_us(caches, qprime, out, torch, device, launches=4000):
    """Microseconds per decode launch: one launch per cache back to back in a
    CUDA graph (no host gaps), the replays bracketed by CUDA events on the
    launching stream; time / launches.  The caches are cycled, so every
    launch reads bytes that the previous ones evicted from L2."""
    stream = torch.cuda.current_stream()
    capture = torch.cuda.Stream(device=device)
    capture.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(capture):
        for c in caches:                      # untimed: attributes, first-use set-up
            c.decode(qprime, out=out, stream=capture)
        capture.synchronize()
        with torch.cuda.graph(graph, stream=capture):
            for c in caches:
                c.decode(qprime, out=out, stream=capture)
    stream.wait_stream(capture)
    reps = max(3, min(200, launches // len(caches)))
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(reps):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    us = g0.elapsed_time(g1) * 1e3 / (reps * len(caches))
    del graph
    return us


def step_graph_time_us(caches, step, dev_pool, i0, torch, device, reps=30):
    """Microseconds per decode step (append + query transform + decode, two
    launches) with one step per cache captured in a CUDA graph, replays
    bracketed by CUDA events.  The capture call appends one token per cache
    (indices i0 .. i0 + copies) after an untimed eager step per cache."""
    stream = torch.cuda.current_stream()
    n = len(caches)
    capture = torch.cuda.Stream(device=device)
    capture.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(capture):
        for i in range(i0, i0 + n):
            step(i, *dev_pool[i % STEP_POOL], stream=capture)
        capture.synchronize()
        with torch.cuda.graph(graph, stream=capture):
            for i in range(i0 + n, i0 + 2 * n):
                step(i, *dev_pool[i % STEP_POOL], stream=capture)
    stream.wait_stream(capture)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(reps):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    us = g0.elapsed_time(g1) * 1e3 / (reps * n)
    del graph
    return us


def run_ours(args, rank, world, device, torch, dist):
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[WORKLOAD]
    bits = args.bits
    stream = torch.cuda.current_stream()
    kd, vd, pool = build_inputs(w, torch, device)
    # set-up steps (one per cache) + warm-up + timed + e2e + the graph timing's
    total_steps = args.copies + args.warmup + args.steps + args.e2e_steps + 2 * args.copies
    grow = math.ceil(total_steps / args.copies) + 8
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, w.context + grow, bits=bits,
                         sink=w.sink, recent=w.recent, chunk=w.chunk)
    caches, Ts, TinvTs = [], [], []
    for c in range(args.copies):
        T, TinvT = I.key_transforms(w, c)
        Ts.append(torch.from_numpy(T).to(device))
        TinvTs.append(torch.from_numpy(TinvT).to(device))
        cache = wk.Cache(cfg, device=device)
        cache.append(kd, vd, Ts[-1])
        caches.append(cache)
    torch.cuda.synchronize()
    del kd, vd
    dev_pool = [tuple(x.to(device) for x in p) for p in pool]
    qprime = torch.empty((w.batch, w.n_q_heads, 128), dtype=torch.float32, device=device)
    out = torch.empty_like(qprime)

    # host-side counts to account the algorithmic bytes of each step
    counts = [c.tokens()[0] for c in caches]

    def step_bytes(i):
        c = i % args.copies
        before = window_state(counts[c], w)
        counts[c] += 1
        after = window_state(counts[c], w)
        dec = decode_bytes(w, bits, after)
        rest = append_bytes(w, bits, after[2] > before[2]) + qtransform_bytes(w)
        return dec, rest

    def step(i, k, v, q, stream=stream, o=None):
        # one call: append 1 token + query transform (one launch) + decode
        c = i % args.copies
        caches[c].decode_step(k, v, Ts[c], q, TinvTs[c], q_prime=qprime, out=out if o is None else o,
                              stream=stream)

    # set-up: every cache (layer) takes one decode step before the warm-up,
    # as in a running server, so that no timed step is the first read of a
    # layer's transforms since its prefill; then W warm-up steps
    i0 = args.copies
    for i in range(i0 + args.warmup):
        step_bytes(i)
        step(i, *dev_pool[i % STEP_POOL])
    torch.cuda.synchronize()

    # ---- timed region: K steps, device resident inputs ----------------------
    K = args.steps
    first = i0 + args.warmup
    dec_total = rest_total = 0
    for i in range(first, first + K):
        d, r = step_bytes(i)
        dec_total += d
        rest_total += r
    counts_after = list(counts)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        # a bounded device-side spin (torch's, ~0.3 ms, untimed) ahead of t0:
        # the host queues the first steps meanwhile, so the timed region
        # starts with work waiting instead of with the first call's enqueue
        torch.cuda._sleep(600_000)
        t0.record(stream)
        h0 = time.perf_counter()
        for i in range(first, first + K):
            step(i, *dev_pool[i % STEP_POOL])
        host_s = time.perf_counter() - h0
        t1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if dist is not None:
        ms = max_over_ranks(ms, dist, device)
    launches_per_step = 2
    status = max(c.device_status() for c in caches)

    # ---- the decode kernel alone (roofline) ------------------------------------
    dec_ms = [decode_graph_us(caches, qprime, out, torch, device) / 1e3]
    dec_launch_bytes = [decode_bytes(w, bits, window_state(counts_after[c], w)) for c in range(args.copies)]
    counts = counts_after

    # ---- the whole step with no host in the loop: one decode_step per cache
    # captured in a CUDA graph (each replay re-appends the captured tokens at
    # the captured positions); minus the decode alone = the step kernel
    step_graph_us = step_graph_time_us(caches, step, dev_pool, first + K, torch, device)
    for i in range(first + K, first + K + 2 * args.copies):
        step_bytes(i)
    e_first = first + K + 2 * args.copies

    # ---- e2e: host buffers, copies inside the timed region --------------------
    # Each step's k, v and q sit back to back in one pinned host buffer: one
    # host->device copy per step (on a copy stream, one step ahead, into one
    # of two device buffers) and one device->host copy of the step's output
    # (on a second copy stream, from one of two output buffers), ordered by
    # events so neither buffer is reused before its copy or step is done.
    E = args.e2e_steps
    NB = 2
    host_outs = [torch.empty((w.batch, w.n_q_heads, 128), dtype=torch.float32).pin_memory() for _ in range(NB)]
    outs = [torch.empty_like(out) for _ in range(NB)]
    e_dec = 0
    for i in range(e_first, e_first + E):
        e_dec += sum(step_bytes(i))
    shapes = [x.shape for x in pool[0]]
    sizes = [x.numel() for x in pool[0]]
    packed = [torch.cat([x.reshape(-1) for x in p]).pin_memory() for p in pool]
    h2d = packed[0].numel() * packed[0].element_size()
    d2h = host_outs[0].numel() * 4
    dbufs = [torch.empty_like(packed[0], device=device) for _ in range(NB)]
    parts = []
    for dbuf in dbufs:
        pb, off = [], 0
        for shp, n in zip(shapes, sizes):
            pb.append(dbuf[off:off + n].view(shp))
            off += n
        parts.append(pb)
    h2d_stream = torch.cuda.Stream(device=device)
    d2h_stream = torch.cuda.Stream(device=device)
    h2d_done = [torch.cuda.Event() for _ in range(NB)]
    step_done = [torch.cuda.Event() for _ in range(NB)]
    d2h_done = [torch.cuda.Event() for _ in range(NB)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()

    def h2d_copy(j):
        b = j % NB
        with torch.cuda.stream(h2d_stream):
            if j >= NB:
                h2d_stream.wait_event(step_done[b])   # step j - NB has read this buffer
            dbufs[b].copy_(packed[(e_first + j) % STEP_POOL], non_blocking=True)
            h2d_done[b].record(h2d_stream)

    e0.record(stream)
    h2d_stream.wait_event(e0)
    if E:
        h2d_copy(0)
    for j in range(E):
        b = j % NB
        if j + 1 < E:
            h2d_copy(j + 1)
        stream.wait_event(h2d_done[b])
        if j >= NB:
            stream.wait_event(d2h_done[b])                # output buffer b has been read back
        step(e_first + j, *parts[b], o=outs[b])
        step_done[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(step_done[b])
            host_outs[b].copy_(outs[b], non_blocking=True)
            d2h_done[b].record(d2h_stream)
    if E:
        stream.wait_event(d2h_done[(E - 1) % NB])
        if E > 1:
            stream.wait_event(d2h_done[(E - 2) % NB])
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    if dist is not None:
        e_ms = max_over_ranks(e_ms, dist, device)

    return dict(w=w, bits=bits, K=K, ms=ms, dec_total=dec_total, rest_total=rest_total, host_s=host_s,
                dec_ms=dec_ms, step_graph_us=step_graph_us, dec_launch_bytes=dec_launch_bytes, clocks=clocks.summary(),
                launches=launches_per_step * K,
                status=status, e2e=(E, e_ms, e_dec, h2d, d2h), copies=args.copies,
                l2_bytes=sum(decode_bytes(w, bits, window_state(c, w)) for c in counts))


PREFILL_WORKLOAD = "qwen3-8b-stack36-b64-prefill32768"


def run_prefill(device, torch, reps=5, batch=0):
    """Bulk append of one layer of the 36-layer workload (batch 64, 32768
    bf16 tokens per sequence, 2-bit percentile-clipped affine): key transform
    on the tensor cores, quantise + pack, values packed.  Each timed append
    goes into a freshly created (zeroed) cache; CUDA events bracket the
    append call alone."""
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[PREFILL_WORKLOAD]
    if batch:
        import dataclasses
        w = dataclasses.replace(w, batch=batch)
    n = w.context
    k, v = I.device_kv(w, 0, n, device=device)
    T, _ = I.key_transforms(w, 0)
    Td = torch.from_numpy(T).to(device)
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, n, bits=2, quantizer=wk.AFFINE_PCTCLIP,
                         sink=w.sink, recent=w.recent, chunk=w.chunk,
                         clip_lo_rank=w.r_lo, clip_hi_rank=w.r_hi)
    buf = torch.empty(wk.cache_bytes(cfg) + 256, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    times = []
    for r in range(reps + 1):
        cache = wk.Cache(cfg, device=device, buffer=buf)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.append(k, v, Td, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        status = cache.device_status()
        cache.close()
        if r > 0:
            times.append(e0.elapsed_time(e1))
    ms = float(np.median(times))
    token_heads = w.batch * n * w.n_kv_heads
    nbytes = token_heads * (2 * 128 * 2 + 2 * (16 * 2 + 4))      # bf16 K, V in; codes + (s, lo) out
    flops = token_heads * 2 * 128 * 128
    peak, src = peaks()
    del k, v, buf
    return {"workload": f"{w.name} (one layer: batch {w.batch}, {n} tokens per sequence, "
                        f"{w.n_kv_heads} KV heads, 2-bit affine ranks {w.r_lo}/{w.r_hi})",
            "ms_per_layer": ms, "tokens_per_s": w.batch * n / (ms / 1e3),
            "token_heads_per_s": token_heads / (ms / 1e3),
            "gbs": nbytes / (ms / 1e3) / 1e9, "frac": nbytes / (ms / 1e3) / 1e9 / peak,
            "key_transform_tflops": flops / (ms / 1e3) / 1e12, "device_status": status,
            "bytes_per_token_head": 2 * 128 * 2 + 2 * (16 * 2 + 4), "peak_source": src,
            "timing": f"median of {reps} appends into a fresh cache, CUDA events"}


def run_workload_decode(name, device, torch, copies, bits=2):
    """Decode throughput of one of the other workloads: `copies` independent
    caches (together larger than L2) filled by one bulk bf16 append through
    the key transform, then decode launches back to back in a CUDA graph."""
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[name]
    n = w.context
    affine = w.quantizer == "affine"
    k, v = I.device_kv(w, 0, n, device=device)
    T, TinvT = I.key_transforms(w, 0)
    Td, TinvTd = torch.from_numpy(T).to(device), torch.from_numpy(TinvT).to(device)
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, n + 128, bits=bits,
                         quantizer=wk.AFFINE_PCTCLIP if affine else wk.QUEST_INT,
                         sink=w.sink, recent=w.recent, chunk=w.chunk,
                         clip_lo_rank=w.r_lo, clip_hi_rank=w.r_hi)
    caches = []
    for _ in range(copies):
        c = wk.Cache(cfg, device=device)
        c.append(k, v, Td)
        caches.append(c)
    del k, v
    qprime = wk.query_transform(I.device_queries(w, 0, 0, device=device), TinvTd)
    out = torch.empty_like(qprime)
    torch.cuda.synchronize()
    us = decode_graph_us(caches, qprime, out, torch, device)
    status = max(c.device_status() for c in caches)
    nbytes = decode_bytes(w, bits, window_state(n, w))
    peak, _ = peaks()
    res = {"workload": f"{name} ({bits}-bit {'affine' if affine else 'QuEST INT'}, G {w.group}, "
                       f"batch {w.batch}, {n} tokens)",
           "decode_us": us, "bytes_per_launch": nbytes, "gbs": nbytes / us / 1e3,
           "frac": nbytes / us / 1e3 / peak, "copies": copies,
           "l2": f"{copies} cycled caches of {nbytes / 1e6:.1f} MB", "device_status": status}
    return res, caches, w, Td


def run_append_steps(caches, w, Td, device, torch, steps=64):
    """One-token appends (key transform, fp16 ring, a chunk flush every
    `chunk` steps) on one cache, each a separate call as a serving loop
    makes them; CUDA events around the whole run."""
    from bit_kv_cache_post_b200 import inputs as I
    cache = caches[0]
    ks, vs = I.device_kv(w, 0, steps, device=device, step=1)
    stream = torch.cuda.current_stream()
    for i in range(4):                       # untimed warm-up of the launch path
        cache.append(ks[:, i:i + 1].contiguous(), vs[:, i:i + 1].contiguous(), Td)
    rows = [(ks[:, i:i + 1].contiguous(), vs[:, i:i + 1].contiguous()) for i in range(4, steps)]
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for kk, vv in rows:
        cache.append(kk, vv, Td)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return {"tokens_per_s": len(rows) * w.batch / (ms / 1e3), "us_per_append": ms * 1e3 / len(rows),
            "appends": len(rows), "flushes": len(rows) // w.chunk, "chunk": w.chunk,
            "device_status": cache.device_status(),
            "timing": "one-token wushkv_append calls back to back, CUDA events around the run"}


def ragged_lengths(w, seed=0):
    """Per-sequence token counts with the workload's mean: pairs context +- d
    with d drawn uniformly from [0, context / 2] (seeded), so the batch holds
    the same number of tokens as the uniform one."""
    g = np.random.default_rng(seed)
    d = g.integers(0, w.context // 2 + 1, size=w.batch // 2)
    n = np.concatenate([w.context + d, w.context - d])
    if w.batch % 2:
        n = np.append(n, w.context)
    return [int(x) for x in g.permutation(n)]


def run_ragged_decode(device, torch, paged: bool, copies=8, bits=2):
    """Decode GB/s of the batch-16 Qwen3-8B-shaped layer when its sequences
    hold different numbers of tokens (ragged_lengths), optionally with the
    packed region paged through a random page table; same total tokens as
    the uniform workload, so the GB/s compare directly."""
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[WORKLOAD]
    lens = ragged_lengths(w)
    nmax = max(lens)
    k, v = I.device_kv(w, 0, nmax, device=device)
    kf = torch.cat([k[b, :n] for b, n in enumerate(lens)]).contiguous()
    vf = torch.cat([v[b, :n] for b, n in enumerate(lens)]).contiguous()
    del k, v
    T, TinvT = I.key_transforms(w, 0)
    Td, TinvTd = torch.from_numpy(T).to(device), torch.from_numpy(TinvT).to(device)
    max_ctx = nmax + 128
    pages_per_seq = (max_ctx + 127) // 128 * 2
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, max_ctx, bits=bits, sink=w.sink,
                         recent=w.recent, chunk=w.chunk,
                         num_pages=w.batch * pages_per_seq if paged else 0)
    caches = []
    for c in range(copies):
        cache = wk.Cache(cfg, device=device)
        if paged:
            perm = np.random.default_rng(100 + c).permutation(cfg.num_pages).astype(np.int32)
            cache.set_page_table(torch.from_numpy(perm.reshape(w.batch, pages_per_seq)).to(device),
                                 pages_per_seq)
        cache.append_varlen(kf, vf, lens, Td)
        caches.append(cache)
    del kf, vf
    qprime = wk.query_transform(I.device_queries(w, 0, 0, device=device), TinvTd)
    out = torch.empty_like(qprime)
    torch.cuda.synchronize()
    us = decode_graph_us(caches, qprime, out, torch, device)
    status = max(c.device_status() for c in caches)
    per_seq = 0
    for n in lens:
        _, ns, P, nr = window_state(n, w)
        per_seq += w.n_kv_heads * (P * 2 * (16 * bits + meta_bytes(w.quantizer)) + (ns + nr) * 2 * 256)
    nbytes = per_seq + 2 * w.batch * w.n_q_heads * 128 * 4
    peak, _ = peaks()
    del caches
    torch.cuda.empty_cache()
    return {"workload": f"{WORKLOAD} with per-sequence lengths {min(lens)}..{max(lens)} "
                        f"(mean {sum(lens) / len(lens):.0f}){', paged packed region' if paged else ''}",
            "lengths": lens, "decode_us": us, "bytes_per_launch": nbytes, "gbs": nbytes / us / 1e3,
            "frac": nbytes / us / 1e3 / peak, "copies": copies, "device_status": status}


def prefill_attention_flops(n, nq, batch, n_q_heads):
    """4 x 128 flop (q.k and p.v) per (query head, visible token); the
    chunk's query i sees n - nq + i + 1 tokens."""
    visible = nq * (n - nq) + nq * (nq + 1) // 2
    return 4.0 * 128 * visible * batch * n_q_heads


def run_prefill_attention(device, torch, nq=512, copies=4, bits=2):
    """Chunked-prefill attention at the batch-16 Qwen3-8B-shaped layer: each
    sequence holds 8192 tokens of which the last nq are the chunk; its
    queries attend causally over the quantised cache.  Launches back to back
    in a CUDA graph over `copies` caches.  Algorithmic flops: 4 x 128 per
    (query head, visible token) (q.k and p.v)."""
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[WORKLOAD]
    n = w.context
    k, v = I.device_kv(w, 0, n, device=device)
    T, TinvT = I.key_transforms(w, 0)
    Td, TinvTd = torch.from_numpy(T).to(device), torch.from_numpy(TinvT).to(device)
    cfg = wk.make_config(w.batch, w.n_kv_heads, w.n_q_heads, n, bits=bits, sink=w.sink,
                         recent=w.recent, chunk=w.chunk)
    caches = []
    for _ in range(copies):
        c = wk.Cache(cfg, device=device)
        c.append(k, v, Td)
        caches.append(c)
    del k, v
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([w.wid, 7]).generate_state(1)[0]))
    q = torch.randn((w.batch * nq, w.n_q_heads, 128), generator=g, device=device).bfloat16()
    qp = wk.query_transform(q, TinvTd).view(w.batch, nq, w.n_q_heads, 128).contiguous()
    out = torch.empty_like(qp)
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream(device=device)
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        for c in caches:
            c.prefill_attention(qp, nq, out=out, stream=cap)
        cap.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            for c in caches:
                c.prefill_attention(qp, nq, out=out, stream=cap)
    stream.wait_stream(cap)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    reps = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
    del graph
    status = max(c.device_status() for c in caches)
    flops = prefill_attention_flops(n, nq, w.batch, w.n_q_heads)
    peak_tf = peaks_tensor()
    tf = flops / us / 1e6
    return {"workload": f"{WORKLOAD}: chunk of the last {nq} of {n} tokens per sequence, {bits}-bit QuEST, G {w.group}",
            "us_per_launch": us, "query_tokens_per_s": w.batch * nq / (us / 1e6),
            "algorithmic_tflops": tf, "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tf[0],
                                                   "unit": "TFLOP/s", "frac": tf / peak_tf[0],
                                                   "peak_source": peak_tf[1]},
            "kernel": "fp16 mma.sync (m16n8k16), scores with the query as hi + lo terms",
            "copies": copies, "device_status": status,
            "timing": "launches back to back in a CUDA graph over the cycled caches, CUDA events"}


def peaks_tensor():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "of measured (MEASURED_PEAKS.json bf16_tflops, burst; fp16 runs at the bf16 rate)"
    except Exception:
        return 1590.0, "of fallback (1.59 PFLOP/s)"


def run_extra(device, torch):
    """Decode GB/s of the 32B-shaped, 4B-shaped long-context and 36-layer
    (one layer, affine) workloads, config-1 decode at 3 and 4 bits, and the
    long-context workload's one-token appends with their 16-token flushes."""
    out = {}
    for name, copies, bits in (("qwen3-32b-layer-b32-ctx32768", 2, 2), ("qwen3-4b-b1-ctx131072", 8, 2),
                               ("qwen3-8b-stack36-b64-prefill32768", 2, 2),
                               ("qwen3-8b-layer-b16-ctx8192", 8, 3), ("qwen3-8b-layer-b16-ctx8192", 8, 4)):
        res, caches, w, Td = run_workload_decode(name, device, torch, copies, bits)
        key = f"{name}_{bits}bit"
        if w.layers > 1:
            res["decode_us_all_layers"] = res["decode_us"] * w.layers
            res["layers"] = w.layers
        if name == "qwen3-4b-b1-ctx131072":
            out["append_" + name] = run_append_steps(caches, w, Td, device, torch)
        out[key] = res
        del caches
        torch.cuda.empty_cache()
    out["prefill_attention_" + WORKLOAD] = run_prefill_attention(device, torch)
    out["ragged_" + WORKLOAD] = run_ragged_decode(device, torch, paged=False)
    out["ragged_paged_" + WORKLOAD] = run_ragged_decode(device, torch, paged=True)
    return out


def run_output_error(device, torch, B=4, n=2048):
    """Module-output-error diagnostic through the library (summary page
    关键实验: relative error of the attention output with the quantised cache,
    geometric mean over (sequence, query head)).  Qwen3-8B-shaped heads with
    the x20 outlier-channel keys, bf16 inputs; transforms: identity, a
    randomised Hadamard rotation, a random invertible T.  The reference is
    exact float64 attention over the same bf16 keys and values, computed with
    plain torch ops."""
    from bit_kv_cache_post_b200 import inputs as I
    from bit_kv_cache_post_b200 import wushkv as wk
    w = I.WORKLOADS[WORKLOAD]
    k = torch.from_numpy(np.stack([I.keys(w, 1, b, n) for b in range(B)])).to(device).bfloat16()
    v = torch.from_numpy(np.stack([I.values(w, 1, b, n) for b in range(B)])).to(device).bfloat16()
    q = torch.from_numpy(np.stack([I.queries(w, 1, b) for b in range(B)])).to(device).bfloat16()
    G = w.group
    # exact reference: softmax(q k^T / sqrt(d)) v per (sequence, query head)
    k64, v64, q64 = k.double(), v.double(), q.double()
    kh = k64.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)          # [B, Hq, n, d]
    vh = v64.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    p = torch.softmax(torch.einsum("bhd,bhnd->bhn", q64, kh) / math.sqrt(128.0), dim=-1)
    ref = torch.einsum("bhn,bhnd->bhd", p, vh)
    arms = {"identity": I.identity_transforms(w), "hadamard": I.hadamard_transforms(w, 1),
            "random_invertible": I.key_transforms(w, 1)}
    table = {}
    for name, (T, TinvT) in arms.items():
        Td, TinvTd = torch.from_numpy(T).to(device), torch.from_numpy(TinvT).to(device)
        for quantizer, qname in ((wk.QUEST_INT, "quest"), (wk.AFFINE_PCTCLIP, "affine")):
            row = {}
            for bits in (2, 3, 4):
                cache = wk.Cache(wk.make_config(B, w.n_kv_heads, w.n_q_heads, n, bits=bits,
                                                quantizer=quantizer), device=device)
                cache.append(k, v, Td)
                out = cache.decode(wk.query_transform(q, TinvTd)).double()
                e = (out - ref).norm(dim=-1) / ref.norm(dim=-1)
                row[f"{bits}bit"] = float(torch.exp(torch.log(e).mean()))
            table[f"{name}_{qname}"] = row
    return {"table": table, "workload": f"{w.name} heads, batch {B}, {n} tokens, bf16, x20 outlier keys",
            "definition": "geometric mean over (sequence, query head) of ||o_quant - o|| / ||o||",
            "pages": "2-bit module-output error on Qwen3-8B: 0.208 (data-adaptive), 0.309 (OSCAR), "
                     "0.325 (Hadamard); context only (needs the model and its data)"}


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_unit(w, bits):
    """Single (sequence 0, KV head 0) oracle cache holding context - 1 tokens
    (untimed set-up) and its step inputs."""
    from bit_kv_cache_post_b200 import inputs as I
    from oracle import wushkv_oracle as O
    n = w.context - 1
    k = I.round_to(I.keys(w, 0, 0, n)[:, :1][None], w.dtype)
    v = I.round_to(I.values(w, 0, 0, n)[:, :1][None], w.dtype)
    T, TinvT = I.key_transform(w, 0, 0)
    oc = O.OracleCache(O.CacheConfig(1, 1, w.group, w.context + 4096, bits=bits,
                                     sink=w.sink, recent=w.recent, chunk=w.chunk))
    oc.append(k, v, T[None].astype(np.float64))
    return oc, T, TinvT


def oracle_step(w, oc, T, TinvT, s, frac=1.0):
    """Append one token, transform the group's queries and decode them over
    the first `frac` of the unit's cached tokens.  Returns algorithmic bytes."""
    from bit_kv_cache_post_b200 import inputs as I
    from oracle import wushkv_oracle as O
    k, v, q = I.step_tokens(w, 0, 0, s % STEP_POOL)
    oc.append(I.round_to(k[:, :1], w.dtype)[None], I.round_to(v[:, :1], w.dtype)[None],
              T[None].astype(np.float64))
    qp = O.transform_query(I.round_to(q[:w.group], w.dtype), TinvT.astype(np.float64))
    ns, P, nr = oc.split()
    if frac >= 1.0:
        oc.decode(qp[None])
        return decode_bytes(w, oc.cfg.bits, (oc.n, ns, P, nr)) // w.units
    # a bounded sample: the same arithmetic over a prefix of the packed tokens
    pt = max(4, int(P * frac)) // 4 * 4
    Kd = O.quest_dequantize(oc.codes_k[0, :pt], oc.meta_k[0, :pt, 0], oc.cfg.bits)
    Vd = O.quest_dequantize(oc.codes_v[0, :pt], oc.meta_v[0, :pt, 0], oc.cfg.bits)
    O.attention_f64(qp, Kd, Vd, 1.0 / math.sqrt(128))
    return pt * 2 * (16 * oc.cfg.bits + meta_bytes(w.quantizer))


def _one_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except Exception:
        class _N:
            def __enter__(self): return self
            def __exit__(self, *a): return False
        return _N()


def cpu_baseline(w, bits, budget_s=15.0):
    from bit_kv_cache_post_b200 import inputs as I  # noqa: F401
    with _one_thread():
        oc, T, TinvT = oracle_unit(w, bits)
        nbytes, reps = 0, 0
        t = time.perf_counter()
        while time.perf_counter() - t < budget_s or reps < 2:
            nbytes += oracle_step(w, oc, T, TinvT, reps)
            reps += 1
        el = time.perf_counter() - t
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"one (sequence, KV head) unit of {w.name}: {reps} steps of 1-token append "
                      f"+ {w.group}-head decode over ~{w.context} tokens, {el:.1f} s, 1 thread"}


def run_reference(args):
    from bit_kv_cache_post_b200 import inputs as I
    w = I.WORKLOADS[WORKLOAD]
    with _one_thread():
        oc, T, TinvT = oracle_unit(w, args.bits)
        t = time.perf_counter()
        oracle_step(w, oc, T, TinvT, 0)
        t_full = time.perf_counter() - t
        frac = min(1.0, 90.0 / max(1, args.steps + args.warmup) / max(t_full, 1e-6))
        for s in range(args.warmup):
            oracle_step(w, oc, T, TinvT, s, frac)
        nbytes = 0
        t = time.perf_counter()
        for s in range(args.steps):
            nbytes += oracle_step(w, oc, T, TinvT, s, frac)
        el = time.perf_counter() - t
    v = nbytes / el / 1e9
    sample = (f"one (sequence, KV head) unit of {w.name}; each step appends 1 token and decodes "
              f"{w.group} heads over {'all' if frac >= 1 else f'{frac:.3%} of the packed'} tokens; 1 thread")
    return {"impl": "reference", "metric": METRIC_NAME, "value": v, "unit": "GB/s",
            "n_gpus": 0, "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(w, args.bits, None),
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

METRIC_NAME = "2-bit KV decode-attention GB/s (% of HBM peak); KV append tokens/s"


DECODE_SOURCES = ["bit_kv_cache_post_b200/csrc/decode.cu", "bit_kv_cache_post_b200/csrc/decode_frag.cuh",
                  "bit_kv_cache_post_b200/csrc/async_copy.cuh",
                  "bit_kv_cache_post_b200/csrc/wushkv_internal.cuh"]


def decode_traffic(bytes_per_launch):
    """DRAM bytes (read + write) of one decode launch, from the committed ncu
    record of this workload, scaled from the captured launch's algorithmic
    bytes to this run's (the traffic grows with the cache bytes); None when
    the decode kernel's sources changed since that capture."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for p in DECODE_SOURCES:
            with open(os.path.join(ROOT, p), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["kernel_sources_sha256"]:
            return None, None
        ratio = rec["traffic_bytes_per_launch"] / rec["algorithmic_bytes_per_launch"]
        return int(round(ratio * bytes_per_launch)), ratio
    except Exception:
        return None, None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "of measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except Exception:
        return 6650.0, "of fallback (6.65 TB/s)"


def config_block(w, bits, copies):
    c = {"workload": w.name, "layers": 1, "batch": w.batch, "n_q_heads": w.n_q_heads,
         "n_kv_heads": w.n_kv_heads, "head_dim": 128, "context": w.context, "bits": bits,
         "quantizer": "QuEST INT", "sink": w.sink, "recent": w.recent, "chunk": w.chunk,
         "input_dtype": w.dtype, "step": "append 1 token/seq + query transform + decode",
         "state": "each cache holds context - 1 prefilled tokens and takes one decode step "
                  "before the warm-up steps"}
    if copies is not None:
        c["l2"] = (f"inputs larger than L2: {copies} independent caches cycled "
                   "(one per layer), ~90 MB of cache bytes each")
    return c


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.only_prefill:
        if rank == 0:
            print(json.dumps({"prefill": run_prefill(device, torch, batch=args.prefill_batch)}))
        if dist is not None:
            dist.destroy_process_group()
        return
    r = run_ours(args, rank, world, device, torch, dist)
    w, bits, K = r["w"], r["bits"], r["K"]
    step_bytes = r["dec_total"] + r["rest_total"]
    value = job_value(step_bytes, r["ms"], world)
    dec_avg_ms = float(np.mean(r["dec_ms"]))
    dec_launch_bytes = float(np.mean(r["dec_launch_bytes"]))
    achieved = dec_launch_bytes / (dec_avg_ms / 1e3) / 1e9
    peak, peak_src = peaks()
    traffic, traffic_ratio = decode_traffic(dec_launch_bytes)
    E, e_ms, e_dec, h2d, d2h = r["e2e"]
    line = {
        "metric": METRIC_NAME, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": r["ms"] / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_block(w, bits, r["copies"]),
        "decode_gbs": world * r["dec_total"] / (r["ms"] / 1e3) / 1e9,
        "append_tokens_per_s": w.batch * K / (r["ms"] / 1e3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "traffic_over_algorithmic": traffic_ratio,
                     "kernel": "decode",
                     "peak_source": peak_src, "frac_of_8tbs": achieved / 8000.0,
                     "launch_ms": dec_avg_ms, "bytes_per_launch": dec_launch_bytes,
                     "timing": "decode launches alone over the same cycled caches after the timed steps: "
                               "one launch per cache back to back in a CUDA graph, CUDA events around the "
                               "replays on the launching stream, time / launches"},
        "e2e": {"value": world * e_dec / (e_ms / 1e3) / 1e9 if E else None,
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": E, "counts": "step bytes / step time incl. each step's pinned host->device input copy and "
                                    "device->host output copy (two copy streams, double-buffered, ordered by "
                                    "events)"},
        "step_breakdown": {"host_enqueue_us_per_step": r["host_s"] * 1e6 / K,
                           "step_us_timed_region": r["ms"] * 1e3 / K,
                           "step_us_graph": r["step_graph_us"],
                           "decode_us": dec_avg_ms * 1e3,
                           "step_kernel_us": r["step_graph_us"] - dec_avg_ms * 1e3,
                           "note": "per step: the step kernel (key append, query transform, chunk flush "
                                   "every 8th step) runs before the decode; step_us_graph is one step per "
                                   "cache in a CUDA graph (no host in the loop), step_kernel_us = "
                                   "step_us_graph - decode_us; the timed region's steps are issued from "
                                   "the host one call at a time"},
        "gpu_launches": r["launches"], "clocks": r["clocks"], "device_status": r["status"],
    }
    if rank == 0 and world == 1 and not args.no_prefill:
        torch.cuda.empty_cache()
        line["prefill"] = run_prefill(device, torch)
    if rank == 0 and world == 1 and not args.no_extra:
        torch.cuda.empty_cache()
        line["workloads"] = run_extra(device, torch)
        line["module_output_error"] = run_output_error(device, torch)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, bits)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


if __name__ == "__main__":
    main()
