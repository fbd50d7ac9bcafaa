"""The multi-GPU path of bench.py on CPU: two gloo ranks (world size 2)
running independent replicas agree on the slowest rank's time and report the
whole-job value."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        out[rank] = (ms, bench.job_value(1e9, ms, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    times = [3.0, 5.0]
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, times, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.0
    # two ranks x 1 GB each over 5 ms
    assert res[0][1] == pytest.approx(2 * 1e9 / 5e-3 / 1e9)
