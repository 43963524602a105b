"""The N-GPU bench path on CPU: world size 2 over gloo.

The layer runs as independent replicas (no collective on the data path); the only
cross-rank step is the timing reduction, which takes the slowest rank's time.  The
reference arm runs on rank 0 only; other ranks exit without work."""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(dist, mine)
        rate = bench.whole_job_rate(64 * 100, world, slowest)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_timing_takes_the_slowest_rank_and_counts_all_ranks_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, rate in out:
        assert slowest == 15.0
        assert rate == pytest.approx(2 * 64 * 100 / 0.015)


def test_single_rank_timing_is_unchanged():
    import bench

    assert bench.max_over_ranks(None, 3.5) == 3.5
    assert bench.whole_job_rate(640, 1, 10.0) == pytest.approx(64000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
