#!/usr/bin/env python
"""Benchmark of the bf16 video-DiT attention forward on B200.

One step = one pass of the whole hot path over the 720p Wan2.1-14B workload:
self-attention (B=1, H=40, Sq=Skv=75,600, D=128, full mask) followed by
cross-attention of the same queries to 512 text tokens.  Inputs are seeded
synthetic tensors (see video_diffusion_transformer_attention_b200/workloads.py),
far larger than L2, resident in HBM before the timed region.

    python bench.py [--gpus N --steps K --warmup W] [--impl vdit|reference]

For N > 1 launch under torch.distributed.run: every rank runs the full
workload on its own GPU (independent problems, no collective on the data
path; "weak" scaling), or with ``--shard heads`` the ranks split the one
problem by heads (strong scaling, still no collective); the time is the max
over ranks.  Rank 0 prints one JSON line.  ``--impl reference`` times the
fp64 CPU oracle on a bounded row sample of the same workload (rank 0 only).
``--all-workloads`` times every workload's calls beside the oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from video_diffusion_transformer_attention_b200 import flops as fl  # noqa: E402
from video_diffusion_transformer_attention_b200 import workloads as wl  # noqa: E402

WORKLOAD = "wan21_14b_720p"
METRIC = "bf16 video-DiT attention fwd TFLOP/s & % of B200 BF16 peak; ms at S=75600"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_lines(text):
    """The source's code without // comments and blank lines: a comment edit
    does not change the kernel the traffic record was taken on."""
    out = []
    for line in text.splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code:
            out.append(code)
    return "\n".join(out)


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("attn_fwd_sm100.cuh", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "video_diffusion_transformer_attention_b200", "csrc", f)) as fh:
            h.update(_code_lines(fh.read()).encode())
    return h.hexdigest()


def recorded_traffic():
    """Per-launch DRAM bytes of the self-attention launch from the committed ncu
    record, or None when the kernel source has changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_sm100_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256") != kernel_source_hash():
        return None
    return float(rec["traffic_per_launch_scaled"])


def workload_config(name):
    w = wl.WORKLOADS[name]
    desc = "; ".join(
        f"{c.name}: B={c.B} H={c.H} Sq={c.Sq} Skv={c.Skv} D={c.D} mask="
        f"{['full', 'block_causal', 'cross', 'block_sparse'][c.mask_kind]}"
        + (f" chunk={c.chunk_tokens}" if c.chunk_tokens else "")
        + (f" density={wl.SPARSE_DENSITY}" if c.mask_kind == wl.MASK_BLOCK_SPARSE else "")
        for c in w.calls)
    return w, desc


# head axis of each input tensor: BSHD tensors on axis 2, the block mask
# [B, H, n_qb, n_kvb] on axis 1
HEAD_AXIS = {"q": 2, "k": 2, "v": 2, "k_text": 2, "v_text": 2, "block_mask": 1}


def cudart():
    """The CUDA runtime already loaded by torch (for pitched async copies)."""
    import ctypes
    for name in ("libcudart.so.12", "/usr/local/cuda/lib64/libcudart.so.12"):
        try:
            rt = ctypes.CDLL(name)
        except OSError:
            continue
        rt.cudaMemcpy2DAsync.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_size_t, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
        rt.cudaMemcpy2DAsync.restype = ctypes.c_int
        return rt
    raise SystemExit("libcudart.so.12 not found")


def copy_heads(rt, dev_t, host_t, axis, h0, hg, upload, stream):
    """Copy heads [h0, h0 + hg) between a pinned host tensor holding every
    head and a compact device tensor holding only those heads, as one
    pitched copy: rows are the dims before the head axis, each row's
    segment the hg heads' contiguous bytes."""
    es = host_t.element_size()
    inner = es
    for n in host_t.shape[axis + 1:]:
        inner *= n
    rows = 1
    for n in host_t.shape[:axis]:
        rows *= n
    H = host_t.shape[axis]
    width, pitch = hg * inner, H * inner
    host_ptr = host_t.data_ptr() + h0 * inner
    if upload:
        err = rt.cudaMemcpy2DAsync(dev_t.data_ptr(), width, host_ptr, pitch, width, rows, 1, stream.cuda_stream)
    else:
        err = rt.cudaMemcpy2DAsync(host_ptr, pitch, dev_t.data_ptr(), width, width, rows, 2, stream.cuda_stream)
    if err != 0:
        raise SystemExit(f"cudaMemcpy2DAsync failed ({err})")


def call_inputs(inp, call):
    if call.mask_kind == wl.MASK_CROSS:
        return inp["q"], inp["k_text"], inp["v_text"]
    return inp["q"], inp["k"], inp["v"]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle legs

def oracle_sample(inp, w, seconds_budget=20.0, seed=0):
    """Time the fp64 oracle on a bounded row sample of every call; TFLOP/s."""
    import oracle
    rng = np.random.default_rng(seed)
    total_flops, total_time, parts = 0.0, 0.0, []
    for call in w.calls:
        q, k, v = call_inputs(inp, call)
        qb, kb, vb = wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v)
        # an equal share of the budget per call, at about 0.5 GFLOP/s per core
        # for this plain fp64 loop
        sparse = call.mask_kind == wl.MASK_BLOCK_SPARSE
        flops_row = 4.0 * call.D * call.Skv * (wl.SPARSE_DENSITY if sparse else 1.0)
        n = int(max(8, min(call.B * call.H * call.Sq,
                          seconds_budget / len(w.calls) * 0.5e9 * oracle.max_threads() / flops_row)))
        rows = np.stack([rng.integers(0, call.B, n), rng.integers(0, call.H, n),
                         rng.integers(0, call.Sq, n)], axis=1)
        mask = inp["block_mask"].numpy() if sparse else None
        t0 = time.perf_counter()
        oracle.attention(qb, kb, vb, call.scale, call.mask_kind, call.chunk_tokens, rows=rows, block_mask=mask)
        dt = time.perf_counter() - t0
        if sparse:
            # exact allowed keys of the sampled rows
            blk = np.minimum(wl.SPARSE_BLOCK, call.Skv - wl.SPARSE_BLOCK * np.arange(mask.shape[-1]))
            keys = (mask[rows[:, 0], rows[:, 1], rows[:, 2] // wl.SPARSE_BLOCK] != 0) @ blk
            f = 4.0 * call.D * float(keys.sum())
        else:
            f = flops_row * n
        total_flops += f
        total_time += dt
        parts.append(f"{call.name}: {n} rows x {call.Skv} keys")
    return total_flops, total_time, "; ".join(parts)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w, desc = workload_config(args.workload)
    inp = wl.workload_inputs(args.workload)
    times, flops_done = [], []
    sample = ""
    # keep the whole --steps/--warmup run within a few minutes of CPU time
    budget = min(args.reference_seconds, 150.0 / max(1, args.warmup + args.steps))
    for s in range(args.warmup + args.steps):
        f, t, sample = oracle_sample(inp, w, seconds_budget=budget, seed=s)
        if s >= args.warmup:
            times.append(t)
            flops_done.append(f)
    value = sum(flops_done) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload} ({desc})", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ rank helpers

def reduce_max(value, dist=None, device="cpu"):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, step_flops, steps, ms):
    """Whole-job throughput: every rank ran `steps` steps of `step_flops` in `ms`."""
    return world * step_flops * steps / (ms * 1e-3) / 1e12


def head_range(H, world, rank):
    """Heads [h0, h1) that rank `rank` of `world` computes when one problem is
    split by heads: contiguous, as even as possible, every head exactly once."""
    h0, h1 = rank * H // world, (rank + 1) * H // world
    if h1 <= h0:
        raise SystemExit(f"--shard heads: {H} heads cannot give each of {world} ranks one")
    return h0, h1


def shard_heads(w, inp, h0, h1):
    """The workload `w` and its CPU inputs restricted to heads [h0, h1).

    (b, h) pairs are independent in the forward, so a rank holding only its
    heads' Q/K/V computes exactly those heads of the full problem with no
    exchange: BSHD tensors are sliced on their head axis (made contiguous, as
    a caller holding head-sharded activations would have them), the block
    mask [B, H, nqb, nkb] on its second axis."""
    import dataclasses
    calls = tuple(dataclasses.replace(c, H=h1 - h0) for c in w.calls)
    out = {}
    for k, t in inp.items():
        out[k] = (t[:, h0:h1] if k == "block_mask" else t[:, :, h0:h1]).contiguous()
    return dataclasses.replace(w, calls=calls), out


# ------------------------------------------------------------------ GPU leg

def run_vdit(args):
    from video_diffusion_transformer_attention_b200 import binding as vb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    vb.lib()
    w, desc = workload_config(args.workload)
    # --qknorm: Q and K are drawn raw; the self-attention call normalises them
    # (per-head RMS norm into a workspace) and then attends
    inp_cpu = wl.workload_inputs(args.workload, raw_qk=args.qknorm)
    # FLOPs of one step of the whole problem (every head)
    problem_flops = sum(fl.attn_flops(c, inp_cpu.get("block_mask")) for c in w.calls)
    heads = None
    H_full = w.calls[0].H
    if args.shard == "heads":
        heads = head_range(w.calls[0].H, world, rank)
        w, inp_cpu = shard_heads(w, inp_cpu, *heads)
    elif args.heads:
        # a smaller case of the same kernels and sequence lengths (for
        # profilers): the first `args.heads` heads of the problem
        if not 0 < args.heads <= w.calls[0].H:
            raise SystemExit(f"--heads {args.heads}: the workload has {w.calls[0].H} heads")
        w, inp_cpu = shard_heads(w, inp_cpu, 0, args.heads)
        problem_flops = sum(fl.attn_flops(c, inp_cpu.get("block_mask")) for c in w.calls)
    inp = {k: v.to(dev) for k, v in inp_cpu.items()}
    outs = []
    for call in w.calls:
        outs.append((torch.empty((call.B, call.Sq, call.H, call.D), dtype=torch.bfloat16, device=dev),
                     torch.empty((call.B, call.H, call.Sq), dtype=torch.float32, device=dev)))
    stream = torch.cuda.Stream(device=dev)
    sptr = int(stream.cuda_stream)
    mask_cpu = inp_cpu.get("block_mask")
    flops_per_call = [fl.attn_flops(c, mask_cpu) for c in w.calls]
    step_flops = sum(flops_per_call)
    qk_ws = None
    if args.qknorm:
        c0 = w.calls[0]
        st, need = vb.vdit_attn_qknorm_plan(c0.B, c0.H, c0.Sq, c0.Skv, c0.D, c0.mask_kind, c0.chunk_tokens)
        if st != vb.VDIT_OK:
            raise SystemExit(f"vdit_attn_qknorm_plan: {vb.vdit_status_string(st)}")
        qk_ws = torch.empty(need, dtype=torch.uint8, device=dev)
    fp8_ws = []
    if args.path == "fp8":
        for c in w.calls:
            st, need = vb.vdit_attn_fp8_plan(c.B, c.H, c.Sq, c.Skv, c.D, c.mask_kind, c.chunk_tokens)
            if st != vb.VDIT_OK:
                raise SystemExit(f"vdit_attn_fp8_plan: {vb.vdit_status_string(st)}")
            fp8_ws.append(torch.empty(need, dtype=torch.uint8, device=dev))
    # kernels of this library launched per call of the step (the 8-bit path's
    # zeroing of its running maxima is a cudaMemsetAsync, not one of these)
    launches_per_call = [(4 if args.path == "fp8" else 1) + (1 if args.qknorm and c.name == "self" else 0)
                         for c in w.calls]

    def launch(i, call, q, k, v, o, lse, mid_event=None, mask=None):
        if args.path == "fp8":
            # quantise (one memset + three kernels), then the 8-bit attention
            ws = fp8_ws[i]
            vb.vdit_fp8_quantize(q, k, v, call.B, call.H, call.Sq, call.Skv, call.D, ws, ws.numel(), sptr)
            if mid_event is not None:
                mid_event.record(stream)
            vb.vdit_attn_fwd_fp8_quantized(o, lse, call.B, call.H, call.Sq, call.Skv, call.D, call.scale,
                                           call.mask_kind, call.chunk_tokens, ws, ws.numel(), sptr)
        elif args.qknorm and call.name == "self":
            vb.vdit_attn_fwd_qknorm(q, k, v, o, lse, None, None, wl.RMS_EPS, call.B, call.H, call.Sq, call.Skv,
                                    call.D, call.scale, call.mask_kind, call.chunk_tokens, qk_ws, qk_ws.numel(),
                                    sptr)
        elif call.mask_kind == wl.MASK_BLOCK_SPARSE:
            vb.vdit_attn_fwd_block_sparse(q, k, v, o, lse, inp["block_mask"] if mask is None else mask, call.B,
                                          call.H, call.Sq, call.Skv, call.D, call.scale, sptr)
        else:
            vb.vdit_attn_fwd(q, k, v, o, lse, call.B, call.H, call.Sq, call.Skv, call.D, call.scale,
                             call.mask_kind, call.chunk_tokens, sptr)

    def step(events=None, inp_set=None, out_set=None):
        inp_set = inp if inp_set is None else inp_set
        out_set = outs if out_set is None else out_set
        for i, call in enumerate(w.calls):
            q, k, v = call_inputs(inp_set, call)
            if events is not None:
                events[i][0].record(stream)
            launch(i, call, q, k, v, *out_set[i], mid_event=events[i][2] if events is not None else None)
            if events is not None:
                events[i][1].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    st, word = vb.vdit_get_device_status(sptr)
    if st != vb.VDIT_OK:
        raise SystemExit(f"device status after warm-up: {vb.vdit_status_string(st)} ({word:#x})")

    per_call_events = [[tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
                        for _ in w.calls] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_start.record(stream)
    for s in range(args.steps):
        step(per_call_events[s])
    t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    call_ms = [statistics.mean(per_call_events[s][i][0].elapsed_time(per_call_events[s][i][1])
                               for s in range(args.steps)) for i in range(len(w.calls))]
    # the attention kernel alone (8-bit path: after the quantisation launches)
    kernel_ms = list(call_ms)
    if args.path == "fp8":
        kernel_ms = [statistics.mean(per_call_events[s][i][2].elapsed_time(per_call_events[s][i][1])
                                     for s in range(args.steps)) for i in range(len(w.calls))]
    st, word = vb.vdit_get_device_status(sptr)
    if st != vb.VDIT_OK:
        raise SystemExit(f"device status after timing: {vb.vdit_status_string(st)} ({word:#x})")
    ms_max = reduce_max(ms, dist, dev)
    ms_per_step = ms_max / args.steps
    # whole-job FLOPs per step: N replicas of the problem, or one problem split by heads
    job_step_flops = problem_flops if heads is not None else world * step_flops
    value = job_tflops(1, job_step_flops, args.steps, ms_max)

    # ---- end to end through the public API, host buffers in and out
    # Every step copies its inputs from pinned host memory and its results
    # back.  Across steps, two device buffer sets per kind and three streams
    # let step i+1's uploads and step i-1's downloads run during step i.  The
    # first and the last step run in G head groups (heads are independent):
    # each group's Q/K/V go up as one pitched copy per tensor into compact
    # [B, S, H/G, D] device buffers, the group's calls run as soon as its
    # inputs have landed, and its O/LSE go down while the next group
    # computes.  Only the first group's upload and the last group's download
    # are exposed.
    e2e = None
    if args.e2e_steps > 0:
        import dataclasses
        H = w.calls[0].H
        # the largest group count up to the requested one that divides H
        G = max(g for g in range(1, max(1, args.e2e_head_groups) + 1) if H % g == 0)
        rt = cudart()
        host_in = {k: v.pin_memory() for k, v in inp_cpu.items()}
        host_out = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(l.shape, dtype=l.dtype).pin_memory())
                    for o, l in outs]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(o.numel() * o.element_size() + l.numel() * l.element_size() for o, l in host_out)
        class BufferSet:
            """Device inputs/outputs of one step, split into `ng` head groups."""

            def __init__(self, ng):
                self.ng, self.hg = ng, H // ng
                self.calls = [dataclasses.replace(c, H=self.hg) for c in w.calls]

                def shape(t, axis):
                    return tuple(self.hg if a == axis else n for a, n in enumerate(t.shape))

                self.inp = [{k: torch.empty(shape(v, HEAD_AXIS[k]), dtype=v.dtype, device=dev) for k, v in inp.items()}
                            for _ in range(ng)]
                self.out = [[(torch.empty(shape(o, 2), dtype=o.dtype, device=dev),
                              torch.empty(shape(l, 1), dtype=l.dtype, device=dev)) for o, l in outs] for _ in range(ng)]
                self.in_ready = [torch.cuda.Event() for _ in range(ng)]
                self.out_ready = [torch.cuda.Event() for _ in range(ng)]
                self.in_free, self.out_free = torch.cuda.Event(), torch.cuda.Event()
                self.used = False

        # Only the first step's uploads and the last step's downloads have no
        # neighbouring compute to hide behind, so those two steps run in head
        # groups; the steps between run whole (one launch per call, no
        # per-group wave tails), their copies overlapping the neighbours'.
        sets = {(g, b): BufferSet(g) for g in sorted({G, 1}) for b in range(2)}
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)

        def pipelined(n_steps):
            for i in range(n_steps):
                bs = sets[(G if i in (0, n_steps - 1) else 1, i % 2)]
                if bs.used:
                    s_in.wait_event(bs.in_free)
                for g in range(bs.ng):
                    for k_, v_ in host_in.items():
                        copy_heads(rt, bs.inp[g][k_], v_, HEAD_AXIS[k_], g * bs.hg, bs.hg, True, s_in)
                    bs.in_ready[g].record(s_in)
                if bs.used:
                    stream.wait_event(bs.out_free)
                for g in range(bs.ng):
                    stream.wait_event(bs.in_ready[g])
                    with torch.cuda.stream(stream):
                        for ci, call in enumerate(bs.calls):
                            q, k, v = call_inputs(bs.inp[g], call)
                            launch(ci, call, q, k, v, *bs.out[g][ci], mask=bs.inp[g].get("block_mask"))
                    bs.out_ready[g].record(stream)
                bs.in_free.record(stream)
                for g in range(bs.ng):
                    s_out.wait_event(bs.out_ready[g])
                    for (o, l), (ho, hl) in zip(bs.out[g], host_out):
                        copy_heads(rt, o, ho, 2, g * bs.hg, bs.hg, False, s_out)
                        copy_heads(rt, l, hl, 1, g * bs.hg, bs.hg, False, s_out)
                bs.out_free.record(s_out)
                bs.used = True

        pipelined(2)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        stream.wait_event(e0)
        s_out.wait_event(e0)
        pipelined(args.e2e_steps)
        e1.record(s_out)
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(e0.elapsed_time(e1), dist, dev)
        # the host results of the last step must equal the device-timed step's
        # results (same inputs; every head is computed independently)
        same = all(torch.equal(ho, o.cpu()) and torch.equal(hl, l.cpu()) for (ho, hl), (o, l) in zip(host_out, outs))
        if not same:
            raise SystemExit("end-to-end results differ from the device-timed step's")
        e2e = {"value": job_tflops(1, job_step_flops, args.e2e_steps, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms / args.e2e_steps, "steps": args.e2e_steps, "head_groups": G,
               "overlap": (f"first and last step in {G} head groups (group g+1 up / g-1 down while group g "
                           "computes); step i+1 up and step i-1 down while step i computes"),
               "results_checked": "host results of the last step equal the device-timed step's, bit for bit"}
        st, word = vb.vdit_get_device_status(sptr)
        if st != vb.VDIT_OK:
            raise SystemExit(f"device status after the end-to-end steps: {vb.vdit_status_string(st)} ({word:#x})")

    line = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        # the self-attention launch dominates the step
        dom = 0
        achieved = flops_per_call[dom] / (kernel_ms[dom] * 1e-3) / 1e12
        # an E4M3 contraction takes twice the bf16 peak (nominal 4.5 vs 2.25 PFLOP/s dense)
        dtype_ratio = 2.0 if args.path == "fp8" else 1.0
        peak_sustained = dtype_ratio * float(peaks.get("bf16_tflops_sustained",
                                                       FALLBACK_PEAKS["bf16_tflops_sustained"]))
        peak_burst = dtype_ratio * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        cross = w.calls[1] if len(w.calls) > 1 else None
        step_bytes = sum(fl.attn_min_bytes(c) for c in w.calls)
        calls = []
        for i, c in enumerate(w.calls):
            calls.append({"call": c.name, "ms": call_ms[i], "tflops": flops_per_call[i] / (call_ms[i] * 1e-3) / 1e12,
                          "hbm_gbs": fl.attn_min_bytes(c) / (call_ms[i] * 1e-3) / 1e9})
            if args.path == "fp8":
                calls[-1]["attention_kernel_ms"] = kernel_ms[i]
                calls[-1]["quantize_ms"] = call_ms[i] - kernel_ms[i]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if heads is not None else "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.path == "fp8" else "bf16", "data": "synthetic",
            "config": {"workload": f"{args.workload} ({desc})" + (" [raw Q/K: per-head RMS norm + attention]"
                                                                  if args.qknorm else "")
                       + (" [8-bit path: E4M3 + V-Smooth + ExpCast-FP8, quantisation inside the step]"
                          if args.path == "fp8" else ""),
                       "l2": f"inputs larger than L2 ({step_bytes / 1e9:.2f} GB of compulsory traffic per step)",
                       **({"heads": f"first {args.heads} of {H_full}"} if args.heads and heads is None else {}),
                       "parallelism": (f"heads split over {world} ranks (rank r: heads [r*H/N, (r+1)*H/N) of "
                                       f"the one problem; rank 0 heads {heads[0]}-{heads[1] - 1}), no collective"
                                       if heads is not None else
                                       f"independent replicas x{world} (no collective)")},
            # The dominant launch is one ~100 ms kernel timed per call with
            # CUDA events, i.e. a kernel timed in isolation: its denominator is
            # the measured burst peak.  The sustained (power-capped) fraction
            # is reported beside it.
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                         "frac": achieved / peak_burst,
                         "traffic": (recorded_traffic() if args.workload == WORKLOAD and args.path == "bf16" and not args.heads
                                     and heads is None else None),
                         "kernel": ("attn_fwd_fp8_sm100_kernel (self-attention launch)" if args.path == "fp8" else
                                    "attn_fwd_sm100_kernel (self-attention launch)" if not args.qknorm else
                                    "qk_rms_norm_kernel + attn_fwd_sm100_kernel (self-attention call)"),
                         "peak_kind": (f"{peak_src} burst bf16 (cuBLAS)" if args.path == "bf16" else
                                       f"2 x {peak_src} burst bf16 (E4M3 at the nominal 2:1 ratio)"),
                         "peak_sustained": peak_sustained,
                         "frac_of_sustained": achieved / peak_sustained,
                         "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS},
            "calls": calls,
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": sum(launches_per_call) * args.steps,
        }
        if cross is not None:
            line["roofline"]["cross_hbm_frac"] = calls[1]["hbm_gbs"] / float(peaks.get("hbm_gbs", 6650.0))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        f, t, sample = oracle_sample(inp_cpu, w, seconds_budget=args.reference_seconds)
        line["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
                                "kind": "oracle", "sample": sample, "seconds": t}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_all_workloads(args):
    """Every workload, one JSON line per attention call: ms/call, algorithmic
    TFLOP/s and its fraction of the measured burst bf16 peak (the cross call
    also in GB/s against the measured copy bandwidth), the median SM clock
    while it ran, and the fp64 oracle timed on the host cores on a row sample
    of the same call (s/row measured, the full call extrapolated from it).

    Each call is timed per launch with CUDA events on its stream, L2 flushed
    (a 256 MB buffer rewritten) before every timed launch; the figure is the
    median over --steps launches after --warmup untimed ones."""
    from video_diffusion_transformer_attention_b200 import binding as vb
    import oracle

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    vb.lib()
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    stream = torch.cuda.Stream(device=dev)
    sptr = int(stream.cuda_stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    cores = oracle.max_threads()
    names = args.workloads.split(",") if args.workloads else list(wl.WORKLOADS)
    for name in names:
        w = wl.WORKLOADS[name]
        inp_cpu = wl.workload_inputs(name)
        inp = {k: v.to(dev) for k, v in inp_cpu.items()}
        mask_cpu = inp_cpu.get("block_mask")
        for call in w.calls:
            q, k, v = call_inputs(inp, call)
            o = torch.empty((call.B, call.Sq, call.H, call.D), dtype=torch.bfloat16, device=dev)
            lse = torch.empty((call.B, call.H, call.Sq), dtype=torch.float32, device=dev)

            def launch():
                if call.mask_kind == wl.MASK_BLOCK_SPARSE:
                    vb.vdit_attn_fwd_block_sparse(q, k, v, o, lse, inp["block_mask"], call.B, call.H, call.Sq,
                                                  call.Skv, call.D, call.scale, sptr)
                else:
                    vb.vdit_attn_fwd(q, k, v, o, lse, call.B, call.H, call.Sq, call.Skv, call.D, call.scale,
                                     call.mask_kind, call.chunk_tokens, sptr)

            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    launch()
            stream.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            clocks = ClockSampler(0)
            clocks.start()
            time.sleep(0.2)
            with torch.cuda.stream(stream):
                for e0, e1 in ev:
                    flush.zero_()
                    e0.record(stream)
                    launch()
                    e1.record(stream)
            stream.synchronize()
            clk = clocks.stop()
            st, word = vb.vdit_get_device_status(sptr)
            if st != vb.VDIT_OK:
                raise SystemExit(f"{name}/{call.name}: device status {vb.vdit_status_string(st)} ({word:#x})")
            times = sorted(e0.elapsed_time(e1) for e0, e1 in ev)
            ms = statistics.median(times)
            flops = fl.attn_flops(call, mask_cpu)
            tflops = flops / (ms * 1e-3) / 1e12
            line = {"workload": name, "call": call.name,
                    "shape": f"B={call.B} H={call.H} Sq={call.Sq} Skv={call.Skv} D={call.D} mask="
                             f"{['full', 'block_causal', 'cross', 'block_sparse'][call.mask_kind]}"
                             + (f" chunk={call.chunk_tokens}" if call.chunk_tokens else ""),
                    "ms": ms, "ms_min": times[0], "ms_max": times[-1], "launches": args.steps,
                    "tflop": flops / 1e12, "tflops": tflops,
                    "frac_of_burst": tflops / burst, "peak_kind": f"{peak_src} burst bf16 {burst} TFLOP/s",
                    "sm_mhz": clk["sm_mhz"], "clock_reasons": clk["reasons"], "l2": "flushed before every launch"}
            if call.mask_kind == wl.MASK_CROSS:
                gbs = fl.attn_min_bytes(call) / (ms * 1e-3) / 1e9
                line["hbm_gbs"] = gbs
                line["hbm_frac"] = gbs / hbm
            # the oracle on a bounded row sample of this call, on the host cores
            qb, kb, vbits = (wl.bf16_bits(t) for t in call_inputs(inp_cpu, call))
            total_rows = call.B * call.H * call.Sq
            density = wl.SPARSE_DENSITY if call.mask_kind == wl.MASK_BLOCK_SPARSE else 1.0
            pairs_per_row = flops / (4.0 * call.D * total_rows)
            n = int(max(8, min(total_rows, args.reference_seconds * 0.5e9 * cores / (4.0 * call.D * call.Skv
                                                                                      * density))))
            rng = np.random.default_rng(0)
            rows = np.stack([rng.integers(0, call.B, n), rng.integers(0, call.H, n),
                             rng.integers(0, call.Sq, n)], axis=1) if n < total_rows else None
            t0 = time.perf_counter()
            oracle.attention(qb, kb, vbits, call.scale, call.mask_kind, call.chunk_tokens, rows=rows,
                             block_mask=mask_cpu.numpy() if mask_cpu is not None else None)
            dt = time.perf_counter() - t0
            rows_done = n if rows is not None else total_rows
            line["oracle"] = {"cores": cores, "rows": rows_done, "seconds": dt, "s_per_row": dt / rows_done,
                              "full_call_s": dt / rows_done * total_rows,
                              "full_call": "extrapolated from the sample" if rows is not None else "measured",
                              "tflops": 4.0 * call.D * pairs_per_row * rows_done / dt / 1e12}
            print(json.dumps(line), flush=True)
            del o, lse
        del inp
        torch.cuda.empty_cache()
    return 0


def run_merge(args):
    """Time vdit_attn_merge at the self-attention shape of the workload (HBM-bound)."""
    from video_diffusion_transformer_attention_b200 import binding as vb
    dev = torch.device("cuda", 0)
    call = wl.WORKLOADS[args.workload].calls[0]
    B, H, S, D = call.B, call.H, call.Sq, call.D
    o_acc = torch.randn(B, S, H, D, device=dev).to(torch.bfloat16)
    o_part = torch.randn(B, S, H, D, device=dev).to(torch.bfloat16)
    lse_acc = torch.randn(B, H, S, device=dev)
    lse_part = torch.randn(B, H, S, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sp = int(stream.cuda_stream)
    for _ in range(args.warmup):
        vb.vdit_attn_merge(o_acc, lse_acc, o_part, lse_part, B, H, S, D, sp)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        vb.vdit_attn_merge(o_acc, lse_acc, o_part, lse_part, B, H, S, D, sp)
    e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    rows = B * H * S
    nbytes = rows * (3 * D * 2 + 3 * 4)  # read two O rows and two LSE, write one of each
    peaks, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"kernel": "attn_merge_kernel", "workload": f"{args.workload} B={B} H={H} S={S} D={D}",
                      "ms": ms, "bytes": nbytes,
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"{src} copy bandwidth"}}),
          flush=True)
    return 0


def run_group(args):
    """Time V-Smooth's Group step (k-means + stable sort) and the K/V gather at the
    self-attention shape of the workload: C clusters seeded from evenly spaced tokens."""
    from video_diffusion_transformer_attention_b200 import binding as vb
    dev = torch.device("cuda", 0)
    call = wl.WORKLOADS[args.workload].calls[0]
    B, H, S, D = call.B, call.H, call.Skv, call.D
    inp = wl.workload_inputs(args.workload)
    k, v = inp["k"].to(dev), inp["v"].to(dev)
    C = args.clusters
    idx = torch.linspace(0, S - 1, C).long()
    cent0 = v[:, idx].float().permute(0, 2, 1, 3).contiguous()  # [B, H, C, D]
    res = {}
    for iters in (0, args.group_iters):
        for _ in range(args.warmup):
            vb.vsmooth_group(v, cent0.clone(), iters=iters)
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            cent = cent0.clone()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            vb.vsmooth_group(v, cent, iters=iters)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        res[iters] = statistics.median(ts)
    _, perm = vb.vsmooth_group(v, cent0.clone(), iters=0)
    for _ in range(args.warmup):
        vb.permute_kv(k, v, perm)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        vb.permute_kv(k, v, perm)
    e1.record()
    torch.cuda.synchronize()
    g_ms = e0.elapsed_time(e1) / args.steps
    st, word = vb.vdit_get_device_status()
    if st != vb.VDIT_OK:
        raise SystemExit(f"device status: {vb.vdit_status_string(st)} ({word:#x})")
    peaks, src = load_peaks()
    nbytes = 4 * B * S * H * D * 2  # K and V read once, written once
    gbs = nbytes / (g_ms * 1e-3) / 1e9
    per_iter = (res[args.group_iters] - res[0]) / max(args.group_iters, 1)
    print(json.dumps({"kernel": "vsmooth_group (assign, accumulate, finalize, sort) + permute_rows_kernel",
                      "workload": f"{args.workload} V: B={B} H={H} S={S} D={D}, C={C}",
                      "assign_and_sort_ms": res[0], "ms_per_lloyd_iteration": per_iter,
                      "assign_gfma": B * H * S * C * D / 1e9,
                      "permute_kv": {"ms": g_ms, "bytes": nbytes, "roofline": {
                          "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"{src} copy bandwidth"}}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("vdit", "reference"), default="vdit")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e-head-groups", type=int, default=8,
                    help="end-to-end leg: split the heads into this many pipelined copy/compute groups "
                         "(the largest divisor of H up to it; 1: whole steps)")
    ap.add_argument("--reference-seconds", type=float, default=40.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", choices=("bf16", "fp8"), default="bf16",
                    help="bf16 attention (default) or the 8-bit path (E4M3 + V-Smooth + ExpCast-FP8)")
    ap.add_argument("--qknorm", action="store_true",
                    help="raw Q/K with the per-head RMS norm fused into the self-attention call")
    ap.add_argument("--kernel", choices=("attention", "merge", "group"), default="attention",
                    help="merge: time only the LSE merge kernel (HBM roofline); group: V-Smooth's Group step "
                         "and the K/V gather")
    ap.add_argument("--clusters", type=int, default=64, help="--kernel group: clusters per head")
    ap.add_argument("--group-iters", type=int, default=1, help="--kernel group: Lloyd iterations")
    ap.add_argument("--heads", type=int, default=0,
                    help="compute only the first N heads of each call (a smaller case of the same kernels)")
    ap.add_argument("--shard", choices=("replicas", "heads"), default="replicas",
                    help="N > 1: every rank runs the whole workload (replicas, weak scaling), or the ranks split "
                         "the one problem by heads (strong scaling, no collective)")
    ap.add_argument("--all-workloads", action="store_true",
                    help="time every workload's calls one by one (one JSON line per call) beside the fp64 oracle "
                         "on a row sample; --workloads picks a comma-separated subset")
    ap.add_argument("--workloads", default="")
    args = ap.parse_args()
    if args.path == "fp8" and args.qknorm:
        ap.error("--qknorm applies to the bf16 path only")
    if args.warmup < 3 and args.impl == "vdit":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.all_workloads:
        return run_all_workloads(args)
    if args.kernel == "merge":
        return run_merge(args)
    if args.kernel == "group":
        return run_group(args)
    return run_vdit(args)


if __name__ == "__main__":
    sys.exit(main())
