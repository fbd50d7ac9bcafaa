"""Failure detection on the GPU without a fault: a decode whose copy waits
run out reports WUSHKV_DEV_TIMEOUT and returns, and the cache stays usable
(needs a B200).

The library's failure injection makes each decode warp's first copy wait on a
barrier that nothing completes, with a limit of a few polls, so it runs out;
the warp then takes its real timeout path and waits at the full limit for its
copies in flight (they land in microseconds), so no copy is outstanding when
the kernel ends.  Nothing here faults, traps or hangs a GPU."""
import numpy as np
import pytest

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


def test_decode_wait_timeout_is_reported_and_recoverable(wk):
    import torch
    n = 64 + 256 + 8 * 40 + 3
    cfg = wk.make_config(2, 2, 8, n, bits=2)
    g = np.random.default_rng(5)
    k = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    v = g.standard_normal((2, n, 2, 128)).astype(np.float32)
    q = g.standard_normal((2, 8, 128)).astype(np.float32)
    cache = wk.Cache(cfg)
    cache.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    qd = torch.from_numpy(q).cuda()
    try:
        wk.inject_decode_timeout(4)
        cache.decode(qd)
        torch.cuda.synchronize()
    finally:
        wk.inject_decode_timeout(0)
    assert cache.device_status(clear=True) & wk.DEV_TIMEOUT
    assert cache.device_status() == 0
    # the next decode on the same cache (and its workspace) is correct
    oc = O.OracleCache(H.oracle_cfg(cfg))
    oc.append(k, v, None)
    out = cache.decode(qd).cpu().numpy()
    want = oc.decode(q.astype(np.float64))
    assert H.rel_rms_err(out, want) <= DECODE_TOL
    assert cache.device_status() == 0
    H.check_guards(cache)
