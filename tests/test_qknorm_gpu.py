"""Fused per-head Q/K RMS norm: raw Q and K in, normalised inside the kernel.

The oracle normalises Q and K in fp64 and rounds them to bf16 (the operand
type of the attention's products); the kernel normalises each tile in fp32 in
shared memory.  An element whose fp32 and fp64 values round to different bf16
neighbours moves by one bf16 ulp, far inside the attention's parity bars.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oracle_attention, rms_norm, round_to_bf16_bits
from tests.helpers import check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


@pytest.mark.parametrize("B,H,Sq,Skv,mask,chunk,weights", [
    (1, 2, 1000, 1000, vb.VDIT_MASK_FULL, 0, False),
    (2, 3, 300, 300, vb.VDIT_MASK_FULL, 0, True),
    (1, 2, 700, 77, vb.VDIT_MASK_CROSS, 0, True),
    (1, 2, 1000, 1000, vb.VDIT_MASK_BLOCK_CAUSAL, 300, False),
])
def test_fused_qknorm_matches_the_oracle_on_normalised_inputs(B, H, Sq, Skv, mask, chunk, weights):
    dev = torch.device("cuda:0")
    q_raw, k_raw, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=71 + Sq, recipe="iid")
    q_raw = (q_raw.float() * 3.0).to(torch.bfloat16)  # raw scale far from 1: the norm must matter
    gen = torch.Generator().manual_seed(5)
    qw = (0.5 + torch.rand(H, 128, generator=gen)) if weights else None
    kw = (0.5 + torch.rand(H, 128, generator=gen)) if weights else None
    eps = 1e-6
    o, lse = vb.attention_qknorm(q_raw.to(dev), k_raw.to(dev), v.to(dev),
                                 None if qw is None else qw.to(dev), None if kw is None else kw.to(dev), eps,
                                 1 / math.sqrt(128), mask, chunk)
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    qn = round_to_bf16_bits(rms_norm(wl.bf16_bits(q_raw), None if qw is None else qw.numpy(), eps))
    kn = round_to_bf16_bits(rms_norm(wl.bf16_bits(k_raw), None if kw is None else kw.numpy(), eps))
    o_r, l_r = oracle_attention(qn, kn, wl.bf16_bits(v), 1 / math.sqrt(128), mask, chunk)
    o_g = o.float().cpu().numpy().astype(np.float64)
    l_g = lse.cpu().numpy().astype(np.float64)
    og = np.concatenate([o_g[b, :, h] for b in range(B) for h in range(H)])
    orr = np.concatenate([o_r[b, :, h] for b in range(B) for h in range(H)])
    groups = [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)]
    res = check_parity(og, orr, l_g.reshape(-1), l_r.reshape(-1), groups, f"qknorm m{mask}",
                       excess_bar=None)  # the kernel attends its own fp32-normalised inputs, the oracle its fp64 ones
    assert res["ok"], res


def test_fused_qknorm_leaves_the_inputs_untouched():
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in wl.draw_qkv(1, 2, 400, 400, 128, seed=72))
    q0, k0 = q.clone(), k.clone()
    vb.attention_qknorm(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(q, q0) and torch.equal(k, k0)


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16).astype(np.int32)


@pytest.mark.parametrize("B,H,Sq,Skv,weights", [
    (1, 3, 37, 5, True),       # 111 + 15 rows: ragged against the 8-row passes
    (2, 40, 300, 512, True),
    (1, 2, 0, 77, False),      # K only
    (1, 5, 1000, 0, True),     # Q only
])
def test_qk_rms_norm_is_within_one_bf16_ulp_of_the_oracle(B, H, Sq, Skv, weights):
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(B * 1000 + Sq + Skv)
    q = (torch.randn(B, Sq, H, 128, generator=g) * 2.5 + 0.3).to(torch.bfloat16)
    k = (torch.randn(B, Skv, H, 128, generator=g) * 0.2).to(torch.bfloat16)
    qw = (0.5 + torch.rand(H, 128, generator=g)) if weights else None
    kw = (0.5 + torch.rand(H, 128, generator=g)) if weights else None
    qo, ko = vb.qk_rms_norm(q.to(dev), k.to(dev), None if qw is None else qw.to(dev),
                            None if kw is None else kw.to(dev), 1e-6)
    torch.cuda.synchronize()
    for x, w, y in ((q, qw, qo), (k, kw, ko)):
        if x.numel() == 0:
            continue
        want = round_to_bf16_bits(rms_norm(wl.bf16_bits(x), None if w is None else w.numpy(), 1e-6))
        got = _bits(y)
        # bf16 patterns of same-sign values are ordered like the values: one step = one ulp
        diff = np.abs(got - want.astype(np.int32))
        assert diff.max() <= 1, diff.max()
        assert (diff != 0).mean() < 0.01


def test_qk_rms_norm_in_place_equals_out_of_place():
    dev = torch.device("cuda:0")
    q, k, _ = (t.to(dev) for t in wl.draw_qkv(1, 4, 999, 640, 128, seed=73))
    w = torch.rand(4, 128, device=dev) + 0.5
    qo, ko = vb.qk_rms_norm(q, k, w, None)
    qi, ki = q.clone(), k.clone()
    vb.qk_rms_norm(qi, ki, w, None, inplace=True)
    torch.cuda.synchronize()
    assert torch.equal(qi, qo) and torch.equal(ki, ko)


@pytest.mark.parametrize("mask,chunk", [(vb.VDIT_MASK_FULL, 0), (vb.VDIT_MASK_BLOCK_CAUSAL, 256)])
def test_chained_entry_equals_norm_then_attention_bitwise(mask, chunk):
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in wl.draw_qkv(1, 3, 1500, 1500, 128, seed=74))
    qw, kw = torch.rand(3, 128, device=dev) + 0.5, torch.rand(3, 128, device=dev) + 0.5
    o1, l1 = vb.attention_qknorm(q, k, v, qw, kw, 1e-6, None, mask, chunk)
    qn, kn = vb.qk_rms_norm(q, k, qw, kw, 1e-6)
    o2, l2 = vb.attention(qn, kn, v, None, mask, chunk)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
