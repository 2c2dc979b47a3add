"""LSE merge kernel: ring context parallelism emulated on one GPU.

K/V are split into uneven shards, each shard is attended separately with the
forward kernel, and the partial results are folded with vdit_attn_merge; the
result must match the oracle over all keys.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oracle_attention
from tests.helpers import check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def test_ring_emulation_matches_the_oracle_over_all_keys():
    dev = torch.device("cuda:0")
    B, H, Sq, D = 2, 3, 700, 128
    shards = [300, 128, 457]
    q, k, v = wl.draw_qkv(B, H, Sq, sum(shards), D, seed=61, recipe="rms_qk")
    qd = q.to(dev)
    scale = 1 / math.sqrt(D)
    o_acc = lse_acc = None
    start = 0
    for n in shards:
        kd = k[:, start:start + n].contiguous().to(dev)
        vd = v[:, start:start + n].contiguous().to(dev)
        o, lse = vb.attention(qd, kd, vd, scale, vb.VDIT_MASK_CROSS)
        if o_acc is None:
            o_acc, lse_acc = o, lse
        else:
            vb.vdit_attn_merge(o_acc, lse_acc, o, lse, B, H, Sq, D)
        start += n
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, vb.VDIT_MASK_CROSS)
    o_g = o_acc.float().cpu().numpy().astype(np.float64)
    l_g = lse_acc.cpu().numpy().astype(np.float64)
    og = np.concatenate([o_g[b, :, h] for b in range(B) for h in range(H)])
    orr = np.concatenate([o_r[b, :, h] for b in range(B) for h in range(H)])
    groups = [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)]
    res = check_parity(og, orr, l_g.reshape(-1), l_r.reshape(-1), groups, "ring emulation",
                       excess_bar=None)  # several partial outputs, each rounded to bf16
    assert res["ok"], res


def test_empty_partials():
    dev = torch.device("cuda:0")
    B, H, S, D = 1, 2, 300, 128
    o = torch.randn(B, S, H, D, device=dev).to(torch.bfloat16)
    lse = torch.randn(B, H, S, device=dev)
    o0, l0 = o.clone(), lse.clone()
    empty_o = torch.randn_like(o)
    empty_l = torch.full_like(lse, float("-inf"))
    vb.vdit_attn_merge(o, lse, empty_o, empty_l, B, H, S, D)
    torch.cuda.synchronize()
    assert torch.equal(o, o0) and torch.allclose(lse, l0, rtol=0, atol=1e-6)
    # both empty: O = 0, LSE = -inf
    a_o, a_l = torch.randn_like(o), torch.full_like(lse, float("-inf"))
    vb.vdit_attn_merge(a_o, a_l, empty_o, empty_l, B, H, S, D)
    torch.cuda.synchronize()
    assert torch.all(a_o == 0) and torch.all(torch.isneginf(a_l))


def test_fp32_running_merge_over_eight_shards():
    """vdit_attn_merge_f32: eight uneven K/V shards folded into an fp32 running
    result that starts at (0, -inf); the last fold also writes the bf16 output,
    which must be the running O rounded to nearest even."""
    dev = torch.device("cuda:0")
    B, H, Sq, D = 1, 3, 640, 128
    shards = [300, 128, 457, 77, 512, 1, 260, 700]
    q, k, v = wl.draw_qkv(B, H, Sq, sum(shards), D, seed=62, recipe="rms_qk")
    qd = q.to(dev)
    scale = 1 / math.sqrt(D)
    o_acc = torch.zeros((B, Sq, H, D), dtype=torch.float32, device=dev)
    lse_acc = torch.full((B, H, Sq), float("-inf"), dtype=torch.float32, device=dev)
    o_out = torch.empty((B, Sq, H, D), dtype=torch.bfloat16, device=dev)
    start = 0
    for i, n in enumerate(shards):
        kd = k[:, start:start + n].contiguous().to(dev)
        vd = v[:, start:start + n].contiguous().to(dev)
        o, lse = vb.attention(qd, kd, vd, scale, vb.VDIT_MASK_CROSS if n <= 512 else vb.VDIT_MASK_FULL)
        vb.vdit_attn_merge_f32(o_acc, lse_acc, o, lse, o_out if i + 1 == len(shards) else None, B, H, Sq, D)
        if i == 0:
            torch.cuda.synchronize()
            assert torch.equal(o_acc, o.float()) and torch.equal(lse_acc, lse)  # the first fold copies exactly
        start += n
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    assert torch.equal(o_out, o_acc.to(torch.bfloat16))
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, vb.VDIT_MASK_CROSS)
    o_g = o_out.float().cpu().numpy().astype(np.float64)
    l_g = lse_acc.cpu().numpy().astype(np.float64)
    og = np.concatenate([o_g[b, :, h] for b in range(B) for h in range(H)])
    orr = np.concatenate([o_r[b, :, h] for b in range(B) for h in range(H)])
    groups = [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)]
    res = check_parity(og, orr, l_g.reshape(-1), l_r.reshape(-1), groups, "fp32 merge, 8 shards",
                       excess_bar=None)  # several partial outputs, each rounded to bf16
    assert res["ok"], res
