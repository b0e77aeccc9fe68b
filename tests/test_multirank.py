"""The N-GPU benchmark path, tested on the CPU with world-size-2 gloo ranks.

The library's collectives run among virtual shards inside one GPU. Several GPUs run independent
replicas, so the only inter-process steps are the barrier and the max-over-ranks reduction of the
timings. Both are exercised here with two gloo processes on 127.0.0.1. The reference arm's
"rank 0 alone runs" rule is checked too.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dist.barrier()
        mine = [10.0 + rank, 5.0 - rank]                 # rank 1 is slower on the first, faster on the second
        got = bench.max_over_ranks(mine, dist)
        rate = bench.whole_job_rate(2.0, 4, world, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    results = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, rate in results:
        assert got == [11.0, 5.0]                        # the slowest rank decides each timing
        assert rate == pytest.approx(2 * 2.0 * 4 / 11e-3)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_rate(1.0, 10, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
