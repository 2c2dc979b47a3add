"""Multi-rank host logic on CPU with gloo (world size 2).

The forward shards with no exchange: each rank runs its own problem and the
benchmark only reduces its timing with a max over ranks.  These tests run that
reduction and the rank handling of the reference arm without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank
        got = bench.reduce_max(mine, dist, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # two ranks, 3 steps of 1 TFLOP each, slowest rank 1.5 s -> 4 TFLOP/s
    assert abs(bench.job_tflops(2, 1e12, 3, 1500.0) - 4.0) < 1e-12
    assert bench.reduce_max(3.5) == 3.5


def test_reference_arm_exits_quietly_on_nonzero_rank():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
