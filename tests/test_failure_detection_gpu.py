"""Failure detection on the GPU without faulting it.

The test-only entry point withholds every K/V tile, so the MMA issuer's
bounded wait on the first K tile runs out.  The kernel must give up, report
VDIT_ERR_TIMEOUT through the device status word, release its resources and
leave the CUDA context usable: a normal call right after it must still match
the oracle.
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

SITE_MMA = 1 << 9


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def test_withheld_kv_times_out_and_context_survives():
    dev = torch.device("cuda:0")
    B, H, S, D = 1, 2, 1000, 128
    q, k, v = wl.draw_qkv(B, H, S, S, D, seed=31, recipe="rms_qk")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK  # clean start
    st = vb.vdit_testing_attn_fwd(qd, kd, vd, o, lse, B, H, S, S, D, 1 / math.sqrt(D), vb.VDIT_MASK_FULL, 0,
                                  vb.VDIT_TESTING_WITHHOLD_KV, 100_000_000)
    assert st == vb.VDIT_OK  # the launch itself succeeds
    st, word = vb.vdit_get_device_status()
    assert st == vb.VDIT_ERR_TIMEOUT
    assert word & 1 and word & SITE_MMA
    assert vb.vdit_get_device_status() == (vb.VDIT_OK, 0)  # reading cleared the word
    # the context is still usable: a normal call afterwards is correct
    o2, lse2 = vb.attention(qd, kd, vd, 1 / math.sqrt(D))
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), 1 / math.sqrt(D))
    o_g = o2.float().cpu().numpy().astype(np.float64)
    res = check_parity(o_g[0].transpose(1, 0, 2).reshape(-1, D), o_r[0].transpose(1, 0, 2).reshape(-1, D),
                       lse2.cpu().numpy().reshape(-1), l_r.reshape(-1), None, "after timeout")
    assert res["ok"], res


def test_cross_attention_over_several_waves_times_out_and_context_survives():
    """The persistent cross launch: every CTA holds several query tiles when the wait runs out."""
    dev = torch.device("cuda:0")
    B, H, Sq, Skv, D = 1, 8, 20000, 512, 128
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, D, seed=33, recipe="rms_qk")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    st = vb.vdit_testing_attn_fwd(qd, kd, vd, o, lse, B, H, Sq, Skv, D, 1 / math.sqrt(D), vb.VDIT_MASK_CROSS, 0,
                                  vb.VDIT_TESTING_WITHHOLD_KV, 100_000_000)
    assert st == vb.VDIT_OK
    st, word = vb.vdit_get_device_status()
    assert st == vb.VDIT_ERR_TIMEOUT
    assert word & 1 and word & SITE_MMA
    assert vb.vdit_get_device_status() == (vb.VDIT_OK, 0)
    o2, lse2 = vb.attention(qd, kd, vd, 1 / math.sqrt(D), vb.VDIT_MASK_CROSS, 0)
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    rows = np.array([0, 1, 255, 256, 9999, 19744, 19999])
    o_r, l_r = oracle_attention(wl.bf16_bits(q[:, rows]), wl.bf16_bits(k), wl.bf16_bits(v), 1 / math.sqrt(D))
    o_g = o2.float().cpu().numpy().astype(np.float64)[:, rows]
    l_g = lse2.cpu().numpy().astype(np.float64)[:, :, rows]
    res = check_parity(o_g[0].transpose(1, 0, 2).reshape(-1, D), o_r[0].transpose(1, 0, 2).reshape(-1, D),
                       l_g.reshape(-1), l_r.reshape(-1), None, "cross, after timeout")
    assert res["ok"], res


def test_testing_entry_point_without_fault_matches_the_product_call():
    dev = torch.device("cuda:0")
    B, H, S, D = 1, 2, 700, 128
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, S, S, D, seed=32, recipe="rms_qk"))
    o1, l1 = vb.attention(q, k, v)
    o2 = torch.empty_like(q)
    l2 = torch.empty_like(l1)
    st = vb.vdit_testing_attn_fwd(q, k, v, o2, l2, B, H, S, S, D, 1 / math.sqrt(D), vb.VDIT_MASK_FULL, 0,
                                  vb.VDIT_TESTING_NO_FAULT, 1_000_000_000)
    assert st == vb.VDIT_OK
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
