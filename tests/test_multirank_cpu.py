"""The multi-replica path of bench.py on the CPU.

bench.py --gpus N runs N independent replicas (one process per GPU, no
collective on the data path).  The only cross-rank steps are barriers and
the maximum of the ranks' device times; here they run on two gloo ranks over
127.0.0.1.  The reference arm is also launched as two ranks the way a
multi-GPU run starts it: rank 0 alone runs and prints, the other exits 0.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        mine = 10.0 + 7.5 * rank          # each rank's own "device time"
        got = bench.max_over_ranks(dist, mine, torch.device("cpu"))
        dist.barrier()
        q.put((rank, mine, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r for r, _, _ in res] == [0, 1]
    assert all(got == 17.5 for _, _, got in res)   # every rank sees the slowest rank's time
    assert all(p.exitcode == 0 for p in procs)


def test_max_over_ranks_without_a_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 3.25, None) == 3.25


@pytest.mark.parametrize("max_ms,calls,world,expect", [
    (10.0, 1000, 1, 10.0),       # one replica: 10 ms over 1000 calls
    (10.0, 1000, 2, 5.0),        # two replicas made 2000 calls in the slowest one's 10 ms
    (0.2, 1, 8, 25.0),
])
def test_whole_job_time_per_call(max_ms, calls, world, expect):
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_us_per_call(max_ms, calls, world) == pytest.approx(expect)


def test_reference_arm_as_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle"
