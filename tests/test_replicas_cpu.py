"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The decode and prefill steps have no exchange between GPUs, so N GPUs run N
replicas; what crosses ranks is the barrier, the maximum of the step times and
the whole-job rate rank 0 reports.  The reference arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.0 + rank                       # rank 1 is the slower one
        dist.barrier()
        worst = bench.rank_max(ms, dist)
        gbs = bench.whole_job_gbs(world, 521_011_200, worst)
        out[rank] = (worst, gbs)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_rate():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        worst, gbs = out[rank]
        assert worst == 2.0                   # the slowest rank's time, on every rank
        assert abs(gbs - 2 * 521_011_200 / 2e-3 / 1e9) < 1e-6


def test_rank_max_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.rank_max(3.5) == 3.5
    assert abs(bench.whole_job_gbs(1, 1e9, 1.0) - 1000.0) < 1e-9


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
