"""Multi-rank host logic on CPU with gloo (world size 2).

The forward shards with no exchange: each rank runs its own problem and the
benchmark only reduces its timing with a max over ranks.  These tests run that
reduction and the rank handling of the reference arm without a GPU.
"""
import json
import math
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


def test_reference_arm_prints_one_contract_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "pr1_s1024", "--steps", "2", "--warmup", "1", "--reference-seconds", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    for key in ("metric", "value", "unit", "n_gpus", "ms_per_step", "higher_is_better", "scaling", "dtype",
                "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


# ---------------------------------------------------------------- context parallel schedules

def _fake_attn(q, k, v):
    """Stand-in for the CUDA attention with Q = 0 semantics: O = mean of the V
    rows, LSE = ln(#keys).  Exercises only the schedule, not the arithmetic."""
    B, Sq, H, D = q.shape
    n = k.shape[1]
    o = v.double().mean(dim=1, keepdim=True).expand(B, Sq, H, D).contiguous()
    lse = torch.full((B, H, Sq), math.log(n), dtype=torch.float64)
    return o, lse


def _fake_merge(o_acc, lse_acc, o_part, lse_part, o_out=None):
    lse = torch.logaddexp(lse_acc, lse_part)
    wa = torch.nan_to_num(torch.exp(lse_acc - lse)).permute(0, 2, 1)[..., None]
    wp = torch.exp(lse_part - lse).permute(0, 2, 1)[..., None]
    o_acc.copy_(wa * o_acc + wp * o_part)
    lse_acc.copy_(lse)
    if o_out is not None:
        o_out.copy_(o_acc)


def _ring_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_attention_b200 import parallel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gen = torch.Generator().manual_seed(7)
        B, S_local, H, D = 1, 5, 3, 8
        v_all = torch.randn(world, B, S_local, H, D, generator=gen, dtype=torch.float64)
        q = torch.zeros(B, 4, H, D, dtype=torch.float64)
        k = torch.zeros(B, S_local, H, D, dtype=torch.float64)
        v = v_all[rank].contiguous()
        o, lse = parallel.ring_attention(q, k, v, attn=_fake_attn, merge=_fake_merge)
        expect = v_all.permute(1, 0, 2, 3, 4).reshape(B, world * S_local, H, D).mean(dim=1)
        out[rank] = (float((o - expect[:, None]).abs().max()), float((lse - math.log(world * S_local)).abs().max()))
    finally:
        dist.destroy_process_group()


def _ulysses_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_attention_b200 import parallel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gen = torch.Generator().manual_seed(3)
        B, S, H, D = 2, 6, 4, 8
        full = torch.randn(B, S, H, D, generator=gen)
        s = S // world
        shard = full[:, rank * s:(rank + 1) * s].contiguous()
        heads = parallel.seq_to_head_shards(shard)
        hs = H // world
        ok_heads = torch.equal(heads, full[:, :, rank * hs:(rank + 1) * hs])
        back = parallel.head_to_seq_shards(heads)
        ok_back = torch.equal(back, shard)
        # full pass with an identity "attention": output = the query shard again
        o, _ = parallel.ulysses_attention(shard, shard, shard, attn=lambda q, k, v: (q, None))
        out[rank] = (ok_heads, ok_back, torch.equal(o, shard))
    finally:
        dist.destroy_process_group()


def _spawn(target, world=2):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    return dict(out)


def test_ring_schedule_visits_every_kv_shard_once():
    out = _spawn(_ring_worker)
    for rank, (err_o, err_lse) in out.items():
        assert err_o < 1e-12 and err_lse < 1e-12, (rank, err_o, err_lse)


def test_ulysses_all_to_all_layouts():
    out = _spawn(_ulysses_worker)
    assert all(all(v) for v in out.values()), out


def _dead_peer_worker(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_attention_b200 import parallel
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left"
        os._exit(0)  # leaves between steps, without tearing down the group
    q = torch.zeros(1, 4, 2, 8, dtype=torch.float64)
    k = torch.zeros(1, 3, 2, 8, dtype=torch.float64)
    v = torch.ones(1, 3, 2, 8, dtype=torch.float64)
    import time
    t0 = time.time()
    try:
        parallel.ring_attention(q, k, v, attn=_fake_attn, merge=_fake_merge)
        out[rank] = "no error"
    except Exception as e:  # the exchange with the departed rank must fail, not hang
        out[rank] = f"error after {time.time() - t0:.1f}s: {type(e).__name__}"


def test_a_departed_rank_makes_the_ring_fail_instead_of_hang():
    out = _spawn(_dead_peer_worker)
    assert out[1] == "left"
    assert out[0].startswith("error after"), out[0]
    assert float(out[0].split()[2][:-2]) < 60


# ---------------------------------------------------------------- one problem split by heads (bench --shard heads)

def _heads_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from video_diffusion_transformer_attention_b200 import flops as fl
    from video_diffusion_transformer_attention_b200 import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for H in (40, 12, 5):
            h0, h1 = bench.head_range(H, world, rank)
            got = [None] * world
            dist.all_gather_object(got, (h0, h1))
            res[H] = got
        # this rank's share of the 720p workload's FLOPs, summed over the ranks
        w = wl.WORKLOADS["wan21_14b_720p"]
        h0, h1 = bench.head_range(w.calls[0].H, world, rank)
        ws, _ = bench.shard_heads(w, {}, h0, h1)
        mine = torch.tensor([sum(fl.attn_flops(c) for c in ws.calls)], dtype=torch.float64)
        dist.all_reduce(mine)
        res["flops"] = float(mine.item())
        # the slices hold exactly this rank's heads
        t = torch.arange(7, dtype=torch.float32).view(1, 1, 7, 1).expand(2, 3, 7, 4).contiguous()
        m = torch.arange(7, dtype=torch.uint8).view(1, 7, 1, 1).expand(2, 7, 3, 3).contiguous()
        h0, h1 = bench.head_range(7, world, rank)
        _, sl = bench.shard_heads(wl.WORKLOADS["pr1_s1024"], {"q": t, "block_mask": m}, h0, h1)
        res["slice"] = (sl["q"][0, 0, :, 0].tolist(), sl["block_mask"][0, :, 0, 0].tolist(),
                        sl["q"].is_contiguous(), list(range(h0, h1)))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_head_split_covers_every_head_once_and_counts_the_whole_problem():
    sys.path.insert(0, ROOT)
    from video_diffusion_transformer_attention_b200 import flops as fl
    from video_diffusion_transformer_attention_b200 import workloads as wl
    out = _spawn(_heads_worker)
    for H in (40, 12, 5):
        ranges = out[0][H]
        assert ranges == out[1][H]
        covered = [h for a, b in ranges for h in range(a, b)]
        assert covered == list(range(H)), (H, ranges)
    assert out[0][40] == [(0, 20), (20, 40)]
    whole = sum(fl.attn_flops(c) for c in wl.WORKLOADS["wan21_14b_720p"].calls)
    assert out[0]["flops"] == whole and out[1]["flops"] == whole
    for rank in (0, 1):
        q_heads, m_heads, contiguous, want = out[rank]["slice"]
        assert q_heads == want and m_heads == want and contiguous
    # strong-scaling throughput: the whole problem's FLOPs over the slowest rank's time
    import bench
    assert abs(bench.job_tflops(1, whole, 2, 100.0) - whole * 2 / 0.1 / 1e12) < 1e-9
