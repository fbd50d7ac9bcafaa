"""The C-ABI library loads and exports every symbol include/wushkv.h declares;
host-only entry points behave (no GPU needed)."""
import ctypes
import os
import re

import pytest

from oracle import wushkv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "wushkv.h")).read()
    return sorted(set(re.findall(r"WUSHKV_API\s+[\w\s\*]+?\b(wushkv_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def wk():
    from bit_kv_cache_post_b200 import build, wushkv
    build.build()
    wushkv.load()
    return wushkv


def test_header_declares_the_api():
    names = _declared()
    assert "wushkv_append" in names and "wushkv_decode" in names and "wushkv_query_transform" in names
    assert len(names) >= 12


def test_library_exports_every_declared_symbol(wk):
    lib = wk.load()
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) >= set(wk.EXPORTED)


def test_default_alpha_matches_oracle(wk):
    """The library computes its own Gaussian-optimal clip ratio; it agrees
    with the oracle's independent computation."""
    for b in (2, 3, 4):
        assert abs(wk.default_quest_alpha(b) - O.quest_alpha(b)) < 1e-12
    assert wk.default_quest_alpha(5) == 0.0


def test_cache_bytes_rejects_bad_configs(wk):
    good = wk.make_config(2, 2, 8, 1000)
    assert wk.cache_bytes(good) > 0
    bad = [
        dict(bits=5), dict(bits=1), dict(n_q_heads=6), dict(n_q_heads=48),
        dict(chunk=6), dict(sink=2), dict(max_ctx=0), dict(quest_alpha=2.5),
        dict(quantizer=1, clip_lo_rank=9), dict(quantizer=1, clip_hi_rank=120),
        dict(quantizer=1, clip_lo_rank=100, clip_hi_rank=100), dict(quantizer=7),
    ]
    for kw in bad:
        base = dict(batch=2, n_kv_heads=2, n_q_heads=8, max_ctx=1000)
        base.update(kw)
        assert wk.cache_bytes(wk.make_config(**base)) == 0, kw
    cfg = wk.make_config(2, 2, 8, 1000)
    cfg.head_dim = 64
    assert wk.cache_bytes(cfg) == 0


def test_cache_bytes_covers_the_packed_bytes(wk):
    """2-bit QuEST: 2 x (32 + 2) bytes per packed token-head plus fp16
    windows, workspace and alignment."""
    cfg = wk.make_config(16, 8, 32, 8192)
    n = wk.cache_bytes(cfg)
    packed = 128 * 8192 * (32 + 32 + 2 + 2)
    windows = 128 * (64 + 264) * 256 * 2
    assert packed + windows < n < 1.2 * (packed + windows)


def test_strerror(wk):
    lib = wk.load()
    assert lib.wushkv_strerror(0) == b"ok"
    assert b"capacity" in lib.wushkv_strerror(2)


def test_null_arguments_are_rejected_without_a_gpu(wk):
    lib = wk.load()
    assert lib.wushkv_append(None, None, None, 0, None, 1, 2, 0, None) == wk.EINVAL
    assert lib.wushkv_decode(None, None, None, 0.0, None) == wk.EINVAL
    assert lib.wushkv_query_transform(None, 0, None, None, 1, 4, 1, None) == wk.EINVAL
    assert lib.wushkv_decode_step(None, None, None, 0, None, None, 0, None, None, None, 0.0, None) == wk.EINVAL
    assert lib.wushkv_decode_noalloc(None, None, None, 0.0, None) == wk.EINVAL
    out = ctypes.c_void_p()
    cfg = wk.make_config(1, 1, 4, 100)
    assert lib.wushkv_cache_create(ctypes.byref(cfg), None, 0, None, ctypes.byref(out)) == wk.EINVAL
