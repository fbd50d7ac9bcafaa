"""The multi-GPU path of bench.py on CPU: two gloo ranks (world size 2)
running independent replicas agree on the slowest rank's time and report the
whole-job value.  The ranks run in a child interpreter so that the test
process itself starts no process group and no worker processes."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import json, os, socket, sys
import torch
import torch.distributed as dist
import torch.multiprocessing as mp
sys.path.insert(0, ROOT)

def rank_main(rank, world, port, times, q):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        q.put((rank, ms, bench.job_value(1e9, ms, world)))
    finally:
        dist.destroy_process_group()

if __name__ == "__main__":
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=rank_main, args=(r, 2, port, [3.0, 5.0], q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=60) for _ in procs)
    for p in procs:
        p.join(60)
    print(json.dumps(res))
'''


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    script = tmp_path / "two_ranks.py"   # spawned ranks re-import it by path
    script.write_text("ROOT = %r\n" % ROOT + SCRIPT)
    r = subprocess.run([sys.executable, str(script)], capture_output=True, text=True, timeout=180,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    import json
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert [x[1] for x in res] == [5.0, 5.0]
    # two ranks x 1 GB each over 5 ms
    assert abs(res[0][2] - 2 * 1e9 / 5e-3 / 1e9) < 1e-6
