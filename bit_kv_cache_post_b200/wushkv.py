"""Python binding of libwushkv.so (argument marshalling only).

Every compute step runs in the library's CUDA kernels; PyTorch supplies
device memory and streams.  Loading fails loudly when the library is
missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwushkv.so")

OK, EINVAL, ECAPACITY, EUNSUPPORTED, ECUDA = range(5)
QUEST_INT, AFFINE_PCTCLIP = 0, 1
F16, BF16, F32 = 0, 1, 2

EXPORTED = [
    "wushkv_cache_bytes", "wushkv_cache_create", "wushkv_cache_destroy", "wushkv_cache_layout",
    "wushkv_cache_tokens", "wushkv_append", "wushkv_query_transform", "wushkv_decode",
    "wushkv_export", "wushkv_device_status", "wushkv_default_quest_alpha", "wushkv_strerror",
    "wushkv_decode_noalloc", "wushkv_decode_step", "wushkv_inject_decode_timeout",
    "wushkv_sequence_tokens", "wushkv_reset_sequence", "wushkv_set_page_table", "wushkv_append_varlen",
    "wushkv_prefill_attention",
]

# bits of the sticky device status word; guard bands after each cache region
DEV_RANGE, DEV_SPLITS, DEV_TIMEOUT = 1, 2, 4
GUARD_BYTES, GUARD_FILL = 256, 0xA5


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "n_kv_heads", "n_q_heads", "head_dim", "max_ctx", "bits",
                 "quantizer", "sink", "recent", "chunk")] + \
               [("quest_alpha", ctypes.c_double),
                ("clip_lo_rank", ctypes.c_int32), ("clip_hi_rank", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


class Layout(ctypes.Structure):
    _fields_ = [
        ("n_planes", ctypes.c_int32), ("plane_bits", ctypes.c_int32 * 2),
        ("packed_capacity", ctypes.c_int32),
        ("k_plane_off", ctypes.c_uint64 * 2), ("v_plane_off", ctypes.c_uint64 * 2),
        ("k_meta_off", ctypes.c_uint64), ("v_meta_off", ctypes.c_uint64),
        ("meta_bytes", ctypes.c_uint32), ("unit_stride", ctypes.c_uint64),
        ("block_stride", ctypes.c_uint64),
        ("sink_k_off", ctypes.c_uint64), ("sink_v_off", ctypes.c_uint64),
        ("sink_unit_stride", ctypes.c_uint64),
        ("ring_k_off", ctypes.c_uint64), ("ring_v_off", ctypes.c_uint64),
        ("ring_unit_stride", ctypes.c_uint64), ("ring_slots", ctypes.c_int32),
        ("workspace_off", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
        ("status_off", ctypes.c_uint64), ("total_bytes", ctypes.c_uint64),
        ("num_pages", ctypes.c_int32), ("page_bytes", ctypes.c_uint64),
    ]


class WushKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_LIB.wushkv_strerror(status).decode() if _LIB else status}")


_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m bit_kv_cache_post_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.wushkv_cache_bytes.argtypes = [ctypes.POINTER(Config)]
    lib.wushkv_cache_bytes.restype = ctypes.c_size_t
    lib.wushkv_cache_create.argtypes = [ctypes.POINTER(Config), vp, ctypes.c_size_t, vp,
                                        ctypes.POINTER(vp)]
    lib.wushkv_cache_destroy.argtypes = [vp]
    lib.wushkv_cache_layout.argtypes = [vp, ctypes.POINTER(Layout)]
    lib.wushkv_cache_tokens.argtypes = [vp] + [ctypes.POINTER(i64)] * 4
    lib.wushkv_append.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, vp]
    lib.wushkv_query_transform.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp]
    lib.wushkv_decode.argtypes = [vp, vp, vp, ctypes.c_float, vp]
    lib.wushkv_decode_noalloc.argtypes = [vp, vp, vp, ctypes.c_float, vp]
    lib.wushkv_prefill_attention.argtypes = [vp, vp, vp, i32, ctypes.c_float, vp]
    lib.wushkv_decode_step.argtypes = [vp, vp, vp, i32, vp, vp, i32, vp, vp, vp, ctypes.c_float, vp]
    lib.wushkv_export.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.wushkv_device_status.argtypes = [vp, i32, ctypes.POINTER(i32)]
    lib.wushkv_sequence_tokens.argtypes = [vp, i32] + [ctypes.POINTER(i64)] * 4
    lib.wushkv_reset_sequence.argtypes = [vp, i32]
    lib.wushkv_set_page_table.argtypes = [vp, vp, i32]
    lib.wushkv_append_varlen.argtypes = [vp, vp, vp, i32, vp, ctypes.POINTER(i32), i32, i32, vp]
    lib.wushkv_inject_decode_timeout.argtypes = [ctypes.c_uint32]
    lib.wushkv_inject_decode_timeout.restype = None
    lib.wushkv_default_quest_alpha.argtypes = [i32]
    lib.wushkv_default_quest_alpha.restype = ctypes.c_double
    lib.wushkv_strerror.argtypes = [i32]
    lib.wushkv_strerror.restype = ctypes.c_char_p
    for name in EXPORTED:
        if name not in ("wushkv_cache_bytes", "wushkv_default_quest_alpha", "wushkv_strerror",
                        "wushkv_inject_decode_timeout"):
            getattr(lib, name).restype = ctypes.c_int32
    _LIB = lib
    return lib


def _check(status: int, what: str):
    if status != OK:
        raise WushKVError(status, what)


_DTYPES = None


def _dtype_code(t) -> int:
    global _DTYPES
    if _DTYPES is None:
        import torch
        _DTYPES = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
    return _DTYPES[t.dtype]


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def make_config(batch, n_kv_heads, n_q_heads, max_ctx, bits=2, quantizer=QUEST_INT, sink=64,
                recent=256, chunk=8, quest_alpha=0.0, clip_lo_rank=2, clip_hi_rank=127,
                num_pages=0) -> Config:
    return Config(batch=batch, n_kv_heads=n_kv_heads, n_q_heads=n_q_heads, head_dim=128,
                  max_ctx=max_ctx, bits=bits, quantizer=quantizer, sink=sink, recent=recent,
                  chunk=chunk, quest_alpha=quest_alpha, clip_lo_rank=clip_lo_rank,
                  clip_hi_rank=clip_hi_rank, num_pages=num_pages)


def cache_bytes(cfg: Config) -> int:
    return int(load().wushkv_cache_bytes(ctypes.byref(cfg)))


def default_quest_alpha(bits: int) -> float:
    return float(load().wushkv_default_quest_alpha(bits))


def inject_decode_timeout(polls: int) -> None:
    """Failure injection for tests: with polls > 0 each decode warp's first
    copy wait runs out after that many polls (0 turns it off)."""
    load().wushkv_inject_decode_timeout(int(polls))


class Cache:
    """One layer's cache over a torch-allocated device buffer."""

    def __init__(self, cfg: Config, device="cuda", stream=None, buffer=None):
        import torch
        lib = load()
        self.cfg = cfg
        nbytes = lib.wushkv_cache_bytes(ctypes.byref(cfg))
        if nbytes == 0:
            raise WushKVError(EINVAL, "invalid cache configuration")
        self.buffer = buffer if buffer is not None else torch.empty(
            nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buffer.data_ptr()
        self._base = (base + 255) // 256 * 256
        self._handle = ctypes.c_void_p()
        _check(lib.wushkv_cache_create(ctypes.byref(cfg), self._base,
                                       nbytes + 256 - (self._base - base),
                                       _stream_ptr(stream), ctypes.byref(self._handle)),
               "wushkv_cache_create")
        self.nbytes = nbytes

    @property
    def handle(self):
        return self._handle

    @property
    def base_ptr(self) -> int:
        return self._base

    def close(self):
        if self._handle:
            load().wushkv_cache_destroy(self._handle)
            self._handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layout(self) -> Layout:
        out = Layout()
        _check(load().wushkv_cache_layout(self._handle, ctypes.byref(out)), "wushkv_cache_layout")
        return out

    def tokens(self, seq: int | None = None) -> tuple[int, int, int, int]:
        """(total, sink, packed, recent) of sequence `seq` (default 0)."""
        v = [ctypes.c_int64() for _ in range(4)]
        _check(load().wushkv_sequence_tokens(self._handle, 0 if seq is None else seq,
                                             *[ctypes.byref(x) for x in v]), "wushkv_sequence_tokens")
        return tuple(int(x.value) for x in v)

    def reset_sequence(self, seq: int):
        _check(load().wushkv_reset_sequence(self._handle, seq), "wushkv_reset_sequence")

    def set_page_table(self, page_table, max_pages_per_seq: int):
        """page_table: [batch][max_pages_per_seq] int32 device tensor (kept
        referenced here so it outlives the cache's use of it)."""
        import torch
        assert page_table.is_contiguous() and page_table.dtype == torch.int32
        self._page_table = page_table
        _check(load().wushkv_set_page_table(self._handle, page_table.data_ptr(), max_pages_per_seq),
               "wushkv_set_page_table")

    def append_varlen(self, k, v, n_new, T=None, stream=None):
        """k, v: [sum(n_new), Hkv, 128] device tensors (sequence 0's tokens,
        then sequence 1's, ...); n_new: per-sequence counts (host)."""
        assert k.is_contiguous() and v.is_contiguous() and k.dtype == v.dtype and k.shape == v.shape
        assert len(n_new) == self.cfg.batch and k.shape[0] == sum(n_new)
        if T is not None:
            assert T.is_contiguous() and T.dtype.itemsize == 4
        counts = (ctypes.c_int32 * len(n_new))(*[int(x) for x in n_new])
        _check(load().wushkv_append_varlen(self._handle, k.data_ptr(), v.data_ptr(), _dtype_code(k),
                                           None if T is None else T.data_ptr(), counts, self.cfg.bits,
                                           self.cfg.quantizer, _stream_ptr(stream)), "wushkv_append_varlen")

    def append(self, k, v, T=None, stream=None, bits=None, quantizer=None):
        """k, v: [B, n_tok, Hkv, 128] device tensors (f16/bf16/f32); T:
        [Hkv, 128, 128] fp32 device tensor or None (keys already transformed)."""
        assert k.is_contiguous() and v.is_contiguous() and k.dtype == v.dtype
        assert k.shape == v.shape and k.shape[0] == self.cfg.batch and k.shape[3] == 128
        if T is not None:
            assert T.is_contiguous() and T.dtype.itemsize == 4
        st = load().wushkv_append(
            self._handle, k.data_ptr(), v.data_ptr(), _dtype_code(k),
            None if T is None else T.data_ptr(), int(k.shape[1]),
            self.cfg.bits if bits is None else bits,
            self.cfg.quantizer if quantizer is None else quantizer, _stream_ptr(stream))
        _check(st, "wushkv_append")

    def decode(self, q_prime, out=None, scale: float = 0.0, stream=None):
        import torch
        assert q_prime.is_contiguous() and q_prime.dtype == torch.float32
        if out is None:
            out = torch.empty_like(q_prime)
        _check(load().wushkv_decode(q_prime.data_ptr(), self._handle, out.data_ptr(), scale,
                                    _stream_ptr(stream)), "wushkv_decode")
        return out

    def decode_step(self, k, v, T, q, TinvT, q_prime=None, out=None, scale: float = 0.0, stream=None):
        """Append one token per sequence (k, v: [B, 1, Hkv, 128]), transform
        the queries (q: [B, Hq, 128]) into q_prime and decode them; returns
        out ([B, Hq, 128] fp32)."""
        import torch
        assert k.is_contiguous() and v.is_contiguous() and q.is_contiguous() and TinvT.is_contiguous()
        assert k.shape == v.shape and k.shape[1] == 1 and T is not None and T.is_contiguous()
        if q_prime is None:
            q_prime = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        _check(load().wushkv_decode_step(self._handle, k.data_ptr(), v.data_ptr(), _dtype_code(k),
                                         T.data_ptr(), q.data_ptr(), _dtype_code(q), TinvT.data_ptr(),
                                         q_prime.data_ptr(), out.data_ptr(), scale, _stream_ptr(stream)),
               "wushkv_decode_step")
        return out

    def prefill_attention(self, q_prime, n_q: int, out=None, scale: float = 0.0, stream=None):
        """Causal attention of the last n_q tokens' queries (q_prime:
        [B, n_q, Hq, 128] fp32, transformed) over the cache; returns out of
        the same shape."""
        import torch
        assert q_prime.is_contiguous() and q_prime.dtype == torch.float32 and q_prime.shape[1] == n_q
        if out is None:
            out = torch.empty_like(q_prime)
        _check(load().wushkv_prefill_attention(q_prime.data_ptr(), self._handle, out.data_ptr(), int(n_q),
                                               scale, _stream_ptr(stream)), "wushkv_prefill_attention")
        return out

    def decode_noalloc(self, q_prime, out=None, scale: float = 0.0, stream=None):
        """As decode(), for callers that cannot allocate device memory: the
        split-K scratch lives in the library's fixed 8 MiB device array."""
        import torch
        assert q_prime.is_contiguous() and q_prime.dtype == torch.float32
        if out is None:
            out = torch.empty_like(q_prime)
        _check(load().wushkv_decode_noalloc(q_prime.data_ptr(), self._handle, out.data_ptr(),
                                            scale, _stream_ptr(stream)), "wushkv_decode_noalloc")
        return out

    def export(self, seq: int, head: int, kv: int, tok0: int, ntok: int):
        """(codes uint8 [ntok,128], meta uint16 [ntok,2], fp16 bits uint16
        [ntok,128], kinds int8 [ntok]) as numpy arrays."""
        import numpy as np
        codes = np.zeros((ntok, 128), np.uint8)
        meta = np.zeros((ntok, 2), np.uint16)
        rows = np.zeros((ntok, 128), np.uint16)
        kinds = np.zeros((ntok,), np.int8)
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        _check(load().wushkv_export(self._handle, seq, head, kv, tok0, ntok, p(codes), p(meta),
                                    p(rows), p(kinds)), "wushkv_export")
        return codes, meta, rows, kinds

    def guard_offsets(self) -> list[int]:
        """Offsets (from the cache base) of the guard bands that follow the
        packed region, sink K, sink V, ring K, ring V and the workspace."""
        L = self.layout()
        U = self.cfg.batch * self.cfg.n_kv_heads
        packed = (L.num_pages + 1) * L.page_bytes if L.num_pages > 0 else U * L.unit_stride
        return [packed, L.sink_k_off + U * L.sink_unit_stride,
                L.sink_v_off + U * L.sink_unit_stride, L.ring_k_off + U * L.ring_unit_stride,
                L.ring_v_off + U * L.ring_unit_stride, L.workspace_off + L.workspace_bytes]

    def device_status(self, clear: bool = False) -> int:
        out = ctypes.c_int32()
        _check(load().wushkv_device_status(self._handle, int(clear), ctypes.byref(out)),
               "wushkv_device_status")
        return int(out.value)


def query_transform(q, TinvT, out=None, n_kv_heads=None, stream=None):
    """q' = T^{-T} q per query head: q [B, Hq, 128] device tensor, TinvT
    [Hkv, 128, 128] fp32 device tensor -> fp32 [B, Hq, 128]."""
    import torch
    assert q.is_contiguous() and TinvT.is_contiguous() and TinvT.dtype == torch.float32
    B, Hq, d = q.shape
    Hkv = TinvT.shape[0] if n_kv_heads is None else n_kv_heads
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _check(load().wushkv_query_transform(q.data_ptr(), _dtype_code(q), TinvT.data_ptr(),
                                         out.data_ptr(), B, Hq, Hkv, _stream_ptr(stream)),
           "wushkv_query_transform")
    return out
