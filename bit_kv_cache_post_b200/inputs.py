"""Seeded synthetic inputs for the WUSH-KV cache path.

This module only draws random numbers with fixed shapes and distributions; it
holds none of the method's arithmetic, so both the CUDA library's callers and
the CPU oracle can use it.  The pages evaluate on Qwen3 checkpoints with
FineWeb-Edu / WikiText-2 data, none of which exists here; these generators
stand in for them with Qwen3 head shapes:

* keys: N(0, 1) post-RoPE keys with per-KV-head outlier channels (chosen
  without replacement, fixed per head) scaled x20 on 8 channels, or x50 on 4
  channels for the 32B-shaped workload;
* values: N(0, 1), or Laplace(0, 1) for the 32B-shaped workload;
* queries: N(0, 1);
* key transform T = c U diag(s) V^T with U, V Haar-orthogonal (QR of a
  Gaussian matrix with the sign fix), s = exp(Uniform(ln 1/4, ln 4)) and c
  chosen so that ||T||_F = sqrt(128); its inverse transpose is
  c^-1 U diag(1/s) V^T in closed form.

Every array comes from ``numpy.random.Generator(PCG64(SeedSequence(...)))``
keyed by (workload id, layer, tensor id, sequence[, step]) so that any
sequence can be regenerated on its own.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128

# tensor ids of the seed scheme
_KEYS, _VALUES, _QUERIES, _TRANSFORM, _OUTLIERS, _STEP_K, _STEP_V, _STEP_Q = range(8)


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # workload id used in the seed scheme
    layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    context: int             # tokens in the cache when the decode query runs
    dtype: str               # "f16" | "bf16" (input dtype of K, V, q)
    bits: tuple[int, ...]
    quantizer: str           # "quest" | "affine"
    sink: int = 64
    recent: int = 256
    chunk: int = 8
    outlier_channels: int = 8
    outlier_scale: float = 20.0
    values: str = "normal"   # "normal" | "laplace"
    r_lo: int = 2
    r_hi: int = 127

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def units(self) -> int:
        return self.batch * self.n_kv_heads


WORKLOADS = {
    w.name: w for w in [
        # tiny single head group, appended then decoded once
        Workload("tiny-gqa4-ctx1024", 0, 1, 1, 4, 1, 1024, "f16", (2,), "quest"),
        # Qwen3-8B-shaped single layer, decode step with one new token
        Workload("qwen3-8b-layer-b16-ctx8192", 1, 1, 16, 32, 8, 8192, "bf16",
                 (2, 3, 4), "quest"),
        # Qwen3-8B-shaped 36-layer stack, prefill 32768 then decode
        Workload("qwen3-8b-stack36-b64-prefill32768", 2, 36, 64, 32, 8, 32768,
                 "bf16", (2,), "affine"),
        # Qwen3-32B-shaped layer, GQA 8, heavier outliers, Laplace values
        Workload("qwen3-32b-layer-b32-ctx32768", 3, 1, 32, 64, 8, 32768, "bf16",
                 (2,), "quest", outlier_channels=4, outlier_scale=50.0,
                 values="laplace"),
        # Qwen3-4B-shaped long context, split-K decode + 16-token chunk flush
        Workload("qwen3-4b-b1-ctx131072", 4, 1, 1, 32, 8, 131072, "bf16", (2,),
                 "quest", chunk=16),
    ]
}


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def outlier_channels(w: Workload, layer: int, head: int) -> np.ndarray:
    return _rng(w.wid, layer, _OUTLIERS, head).choice(
        HEAD_DIM, size=w.outlier_channels, replace=False)


def _key_scale(w: Workload, layer: int) -> np.ndarray:
    sc = np.ones((w.n_kv_heads, HEAD_DIM), np.float32)
    for h in range(w.n_kv_heads):
        sc[h, outlier_channels(w, layer, h)] = w.outlier_scale
    return sc


def keys(w: Workload, layer: int, seq: int, n: int) -> np.ndarray:
    """First ``n`` post-RoPE keys of sequence ``seq``: [n, Hkv, 128] float32."""
    x = _rng(w.wid, layer, _KEYS, seq).standard_normal((n, w.n_kv_heads, HEAD_DIM),
                                                       dtype=np.float32)
    return x * _key_scale(w, layer)[None]


def values(w: Workload, layer: int, seq: int, n: int) -> np.ndarray:
    """First ``n`` values of sequence ``seq``: [n, Hkv, 128] float32."""
    g = _rng(w.wid, layer, _VALUES, seq)
    shape = (n, w.n_kv_heads, HEAD_DIM)
    if w.values == "laplace":
        return g.laplace(0.0, 1.0, shape).astype(np.float32)
    return g.standard_normal(shape, dtype=np.float32)


def step_tokens(w: Workload, layer: int, seq: int, step: int):
    """(k [1, Hkv, 128], v [1, Hkv, 128], q [Hq, 128]) for decode step ``step``."""
    k = _rng(w.wid, layer, _STEP_K, seq, step).standard_normal(
        (1, w.n_kv_heads, HEAD_DIM), dtype=np.float32) * _key_scale(w, layer)[None]
    g = _rng(w.wid, layer, _STEP_V, seq, step)
    if w.values == "laplace":
        v = g.laplace(0.0, 1.0, (1, w.n_kv_heads, HEAD_DIM)).astype(np.float32)
    else:
        v = g.standard_normal((1, w.n_kv_heads, HEAD_DIM), dtype=np.float32)
    q = _rng(w.wid, layer, _STEP_Q, seq, step).standard_normal(
        (w.n_q_heads, HEAD_DIM), dtype=np.float32)
    return k, v, q


def queries(w: Workload, layer: int, seq: int) -> np.ndarray:
    """[Hq, 128] float32 decode query of sequence ``seq``."""
    return _rng(w.wid, layer, _QUERIES, seq).standard_normal(
        (w.n_q_heads, HEAD_DIM), dtype=np.float32)


def _haar(g: np.random.Generator, d: int) -> np.ndarray:
    a = g.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def key_transform(w: Workload, layer: int, head: int) -> tuple[np.ndarray, np.ndarray]:
    """(T, T^{-T}) for one KV head, float32 [128, 128] row-major."""
    g = _rng(w.wid, layer, _TRANSFORM, head)
    U, V = _haar(g, HEAD_DIM), _haar(g, HEAD_DIM)
    s = np.exp(g.uniform(np.log(0.25), np.log(4.0), HEAD_DIM))
    c = np.sqrt(HEAD_DIM) / np.linalg.norm(s)
    T = c * (U * s[None, :]) @ V.T
    TinvT = (1.0 / c) * (U * (1.0 / s)[None, :]) @ V.T
    return T.astype(np.float32), TinvT.astype(np.float32)


_HADAMARD_SIGNS = 8   # tensor id of the seed scheme (random signs of the rotation)


def _sylvester(d: int) -> np.ndarray:
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_transform(w: Workload, layer: int, head: int) -> tuple[np.ndarray, np.ndarray]:
    """(T, T^{-T}) of a randomised Hadamard rotation for one KV head: the
    Sylvester Hadamard matrix scaled by 1/sqrt(128) times a diagonal of
    seeded random signs (orthogonal, so T^{-T} = T).  The data-independent
    rotation the pages compare against."""
    signs = _rng(w.wid, layer, _HADAMARD_SIGNS, head).choice([-1.0, 1.0], HEAD_DIM)
    T = (_sylvester(HEAD_DIM) / np.sqrt(HEAD_DIM)) * signs[None, :]
    return T.astype(np.float32), T.astype(np.float32)


def hadamard_transforms(w: Workload, layer: int) -> tuple[np.ndarray, np.ndarray]:
    pairs = [hadamard_transform(w, layer, h) for h in range(w.n_kv_heads)]
    return np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs])


def identity_transforms(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    eye = np.broadcast_to(np.eye(HEAD_DIM, dtype=np.float32), (w.n_kv_heads, HEAD_DIM, HEAD_DIM))
    return np.ascontiguousarray(eye), np.ascontiguousarray(eye)


def key_transforms(w: Workload, layer: int) -> tuple[np.ndarray, np.ndarray]:
    """(T [Hkv,128,128], T^{-T} [Hkv,128,128]) float32."""
    pairs = [key_transform(w, layer, h) for h in range(w.n_kv_heads)]
    return np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs])


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the workload's input dtype, returned as
    float32 (what both sides then read)."""
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float32)
    if dtype == "bf16":
        u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
        # round to nearest even on the upper 16 bits (finite inputs)
        r = ((u >> 16) & 1) + np.uint32(0x7FFF)
        return ((u + r) & np.uint32(0xFFFF0000)).view(np.float32)
    if dtype == "f32":
        return np.asarray(x, np.float32)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Device-side draws for the workloads too large to generate on the host.
# Same distributions (outlier channels are the host generator's), drawn with
# torch's seeded CUDA generator; tests copy back the sampled units so that the
# oracle reads exactly the values the library received.
# ---------------------------------------------------------------------------

def device_kv(w: Workload, layer: int, n: int, device="cuda", step: int | None = None,
              dtype=None):
    """(k, v) of all sequences: [B, n, Hkv, 128] tensors in the workload's
    dtype (or `dtype`), drawn on `device`.  `step` selects an independent
    stream (per decode step)."""
    import torch
    tdt = dtype or {"bf16": torch.bfloat16, "f16": torch.float16}[w.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([w.wid, layer, _KEYS, 0 if step is None else step + 1])
                      .generate_state(1)[0]))
    k = torch.randn((w.batch, n, w.n_kv_heads, HEAD_DIM), generator=g, device=device)
    k *= torch.from_numpy(_key_scale(w, layer)).to(device)[None, None]
    if w.values == "laplace":
        u = torch.rand((w.batch, n, w.n_kv_heads, HEAD_DIM), generator=g, device=device) - 0.5
        v = -torch.sign(u) * torch.log1p(-2.0 * u.abs().clamp_max(0.5 - 2.0 ** -25))
    else:
        v = torch.randn((w.batch, n, w.n_kv_heads, HEAD_DIM), generator=g, device=device)
    return k.to(tdt), v.to(tdt)


def device_queries(w: Workload, layer: int, step: int, device="cuda", dtype=None):
    """[B, Hq, 128] decode queries drawn on `device`."""
    import torch
    tdt = dtype or {"bf16": torch.bfloat16, "f16": torch.float16}[w.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([w.wid, layer, _QUERIES, step]).generate_state(1)[0]))
    return torch.randn((w.batch, w.n_q_heads, HEAD_DIM), generator=g, device=device).to(tdt)
