"""Host logic of the multi-GPU (replica) bench path on CPU: two gloo ranks, the job time is
the max over ranks, the job throughput counts every rank's units, and the reference arm runs
on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        t_ms = 10.0 + 5.0 * rank            # rank 1 is the slowest
        job_ms = bench.reduce_max(t_ms, world, "cpu")
        q.put((rank, job_ms, bench.job_throughput(64 * 256, world, job_ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, job_ms, value in res:
        assert job_ms == 15.0
        assert abs(value - 2 * 64 * 256 / 15e-3) < 1e-6 * value


def test_reference_arm_is_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_single_rank_reduction_is_identity():
    assert bench.reduce_max(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(100, 1, 1000.0) == 100.0
