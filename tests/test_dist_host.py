"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

The layer shards over tokens with no exchange, so the only cross-rank
operations are the barrier and the max-over-ranks of the elapsed time; both
are exercised here with two processes on the host."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        elapsed = [12.5, 40.25][rank]          # each rank's own device time (ms)
        mx = bench.max_over_ranks(elapsed, world)
        val = bench.weak_scaling_value(2.0e12, 10, world, mx)
        q.put((rank, mx, val))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, val in res:
        assert mx == 40.25                                   # the slowest rank's time
        assert val == pytest.approx(2.0e12 * 10 * 2 / 40.25e-3 / 1e12)   # all ranks' work / that time


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.dist_setup() == (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                                  int(os.environ.get("LOCAL_RANK", "0")))


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
