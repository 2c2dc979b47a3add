"""Ring and Ulysses context parallelism with the CUDA kernels, on one GPU.

The Wave Forcing digest (airadar.tv) compares its Wave Parallelism with
Ulysses (all-to-all from sequence shards to head shards and back) and Ring
context parallelism (K/V blocks passed around a ring, partial results merged
through their log-sum-exp).  ``parallel.ring_attention`` and
``parallel.ulysses_attention`` run here exactly as a user calls them -- the
default attention (``vdit_attn_fwd``) and merge (``vdit_attn_merge_f32``) --
on gloo ranks that are separate processes sharing cuda:0.  Gloo carries CPU
tensors only, so the schedules stage their CUDA shards through host memory;
the kernels of one rank never wait on another rank's, only the host-side
exchange does.  Each rank's O and LSE are compared with the fp64 oracle over
the whole, unsharded sequence under the parity checker's bars.
"""
import datetime
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import attention as oracle_attention
from tests.helpers import check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FULL, BC = vb.VDIT_MASK_FULL, vb.VDIT_MASK_BLOCK_CAUSAL


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, kind, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from video_diffusion_transformer_attention_b200 import binding as vb_
    from video_diffusion_transformer_attention_b200 import parallel
    from video_diffusion_transformer_attention_b200 import workloads as wl_
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        dev = torch.device("cuda:0")
        B, H, S, mask, chunk, seed = case
        q, k, v = wl_.draw_qkv(B, H, S, S, 128, seed=seed, recipe="rms_qk")
        s = S // world
        shard = [t[:, rank * s:(rank + 1) * s].contiguous().to(dev) for t in (q, k, v)]
        if kind == "ring":
            o, lse = parallel.ring_attention(*shard)
        else:
            o, lse = parallel.ulysses_attention(*shard, mask_kind=mask, chunk_tokens=chunk)
        torch.cuda.synchronize()
        st, word = vb_.vdit_get_device_status()
        out[rank] = (o.float().cpu().numpy(), lse.float().cpu().numpy(), st, word)
    finally:
        dist.destroy_process_group()


def _run(kind, world, case):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, kind, case, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    return dict(out)


RING = [  # world, (B, H, S, mask, chunk, seed): shards of S / world keys
    (2, (1, 3, 2048, FULL, 0, 71)),   # 1024-key shards: the full kernel
    (4, (2, 2, 1500, FULL, 0, 72)),   # 375-key shards (ragged): the short-key kernel
    (8, (1, 2, 4096, FULL, 0, 73)),   # eight folds into the fp32 running result
]


@pytest.mark.parametrize("world,case", RING)
def test_ring_attention_with_the_cuda_kernels(world, case):
    B, H, S, mask, chunk, seed = case
    out = _run("ring", world, case)
    q, k, v = wl.draw_qkv(B, H, S, S, 128, seed=seed, recipe="rms_qk")
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), 1 / math.sqrt(128), mask, chunk)
    s = S // world
    for rank in range(world):
        o, lse, st, word = out[rank]
        assert st == vb.VDIT_OK, (rank, vb.vdit_status_string(st), hex(word))
        og = np.concatenate([o[b, :, h] for b in range(B) for h in range(H)])
        orr = np.concatenate([o_r[b, rank * s:(rank + 1) * s, h] for b in range(B) for h in range(H)])
        lg = np.concatenate([lse[b, h] for b in range(B) for h in range(H)])
        lr = np.concatenate([l_r[b, h, rank * s:(rank + 1) * s] for b in range(B) for h in range(H)])
        groups = [np.arange(i * s, (i + 1) * s) for i in range(B * H)]
        res = check_parity(og, orr, lg, lr, groups, f"ring N={world} rank {rank}",
                           excess_bar=None)  # N partial outputs, each rounded to bf16, merged
        assert res["ok"], res


ULYSSES = [  # world, (B, H, S, mask, chunk, seed)
    (2, (1, 4, 1500, FULL, 0, 74)),
    (2, (2, 4, 1500, BC, 300, 75)),   # block-causal: every rank sees whole sequences of its heads
    (4, (1, 8, 2048, BC, 700, 76)),
]


@pytest.mark.parametrize("world,case", ULYSSES)
def test_ulysses_attention_with_the_cuda_kernels(world, case):
    B, H, S, mask, chunk, seed = case
    out = _run("ulysses", world, case)
    q, k, v = wl.draw_qkv(B, H, S, S, 128, seed=seed, recipe="rms_qk")
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), 1 / math.sqrt(128), mask, chunk)
    s, hs = S // world, H // world
    for rank in range(world):
        o, lse, st, word = out[rank]
        assert st == vb.VDIT_OK, (rank, vb.vdit_status_string(st), hex(word))
        assert o.shape == (B, s, H, 128) and lse.shape == (B, hs, S)
        # O: this rank's sequence shard, every head
        og = np.concatenate([o[b, :, h] for b in range(B) for h in range(H)])
        orr = np.concatenate([o_r[b, rank * s:(rank + 1) * s, h] for b in range(B) for h in range(H)])
        groups = [np.arange(i * s, (i + 1) * s) for i in range(B * H)]
        res = check_parity(og, orr, None, None, groups, f"ulysses N={world} rank {rank} O")
        assert res["ok"], res
        # LSE: this rank's heads, every token
        lg = lse.reshape(-1)
        lr = np.concatenate([l_r[b, rank * hs + j] for b in range(B) for j in range(hs)])
        assert np.max(np.abs(lg - lr) / np.maximum(np.abs(lr), 1.0)) <= 1e-3
