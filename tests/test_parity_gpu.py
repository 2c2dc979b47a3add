"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle.

Small shapes compare every output element; they span several 128-row tiles,
ragged tails, chunk boundaries inside tiles and degenerate lengths.  The five
workload shapes at full size compare a deterministic row sample (every head,
tile and chunk boundary rows, seeded-random rows), each row computed by the
oracle over all of its allowed keys.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oracle_attention
from tests.helpers import check_parity, round_bf16
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu

FULL, BC, CROSS = vb.VDIT_MASK_FULL, vb.VDIT_MASK_BLOCK_CAUSAL, vb.VDIT_MASK_CROSS


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def run_gpu(q, k, v, scale, mask_kind, chunk=0):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = vb.attention(qd, kd, vd, scale, mask_kind, chunk)
    st, word = vb.vdit_get_device_status()
    assert st == vb.VDIT_OK, f"device status {vb.vdit_status_string(st)} word={word:#x}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def compare_all_rows(q, k, v, scale, mask_kind, chunk=0, label=""):
    o_g, l_g = run_gpu(q, k, v, scale, mask_kind, chunk)
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, mask_kind, chunk)
    B, Sq, H, D = q.shape
    groups, og, orr, lg, lr = [], [], [], [], []
    n = 0
    for b in range(B):
        for h in range(H):
            og.append(o_g[b, :, h]); orr.append(o_r[b, :, h])
            lg.append(l_g[b, h]); lr.append(l_r[b, h])
            groups.append(np.arange(n, n + Sq)); n += Sq
    res = check_parity(np.concatenate(og), np.concatenate(orr), np.concatenate(lg), np.concatenate(lr),
                       groups, label)
    assert res["ok"], res
    return res


SMALL_CASES = [
    # B, H, Sq, Skv, mask, chunk, recipe
    (1, 2, 1024, 1024, FULL, 0, "iid"),          # the small reference workload
    (1, 2, 1, 1, FULL, 0, "iid"),
    (1, 1, 7, 7, FULL, 0, "iid"),
    (1, 2, 127, 127, FULL, 0, "rms_qk"),
    (1, 2, 128, 128, FULL, 0, "rms_qk"),
    (1, 2, 129, 129, FULL, 0, "rms_qk"),
    (1, 1, 255, 255, FULL, 0, "iid"),
    (1, 1, 256, 256, FULL, 0, "iid"),
    (2, 3, 300, 300, FULL, 0, "rms_qk_vout"),
    (1, 2, 777, 777, FULL, 0, "rms_qk"),
    (1, 2, 300, 512, CROSS, 0, "iid"),
    (1, 3, 1000, 77, CROSS, 0, "iid"),
    (1, 2, 5, 1000, CROSS, 0, "iid"),
    (1, 2, 333, 1, CROSS, 0, "iid"),
    (1, 2, 1000, 1000, BC, 100, "rms_qk"),
    (1, 2, 777, 777, BC, 130, "rms_qk"),
    (1, 1, 513, 513, BC, 1, "iid"),
    (1, 2, 600, 600, BC, 600, "iid"),
    (1, 2, 600, 600, BC, 5000, "iid"),
    (2, 2, 1024, 1024, BC, 256, "rms_qk"),
    (1, 1, 9360, 9360, BC, 4680, "rms_qk"),
]


@pytest.mark.parametrize("B,H,Sq,Skv,mask,chunk,recipe", SMALL_CASES)
def test_parity_all_rows(B, H, Sq, Skv, mask, chunk, recipe):
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=7 + Sq + Skv + H, recipe=recipe)
    compare_all_rows(q, k, v, 1 / math.sqrt(128), mask, chunk, f"{B}x{H}x{Sq}x{Skv} m{mask} c{chunk}")


# Cross attention runs persistently, two CTAs per SM taking 128-row query
# tiles in turn: with more tiles than CTAs each CTA takes several, reloading Q
# between them while its K/V ring carries on.  Every row compared: short text
# sequences of one to four key tiles, ragged query and key tails, batch > 1.
WIDE_CROSS = [
    # B, H, Sq, Skv
    (2, 5, 9000, 77),      # one key tile
    (1, 4, 20000, 300),    # three key tiles, ragged query and key tails
    (1, 40, 9000, 130),    # about ten waves of CTAs, two key tiles
    (1, 3, 30000, 512),    # the text length of the 720p workload
]


@pytest.mark.parametrize("B,H,Sq,Skv", WIDE_CROSS)
def test_cross_attention_over_several_waves(B, H, Sq, Skv):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert B * H * -(-Sq // 128) > 2 * sms  # more query tiles than CTAs
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=41 + Sq + Skv, recipe="rms_qk")
    compare_all_rows(q, k, v, 1 / math.sqrt(128), CROSS, 0, f"cross {B}x{H}x{Sq}x{Skv}")


def test_cross_attention_runs_two_ctas_per_sm():
    """The persistent cross-attention grid is two CTAs per SM, which the
    occupancy query does not confirm for this kernel: the CTAs record the SM
    they ran on and their lifetimes, and every SM must hold two of them at the
    same time.  The recording call's output is the product call's, bit for bit."""
    from collections import Counter
    dev = torch.device("cuda:0")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, H, Sq, Skv = 1, 40, 20000, 512
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, Sq, Skv, 128, seed=43, recipe="rms_qk"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
    spans = torch.zeros((4 * sms, 3), dtype=torch.int64, device=dev)
    st, grid = vb.vdit_testing_cross_cta_spans(q, k, v, o, lse, B, H, Sq, Skv, 128, 1 / math.sqrt(128), spans,
                                               4 * sms)
    assert st == vb.VDIT_OK, vb.vdit_status_string(st)
    assert vb.vdit_get_device_status()[0] == vb.VDIT_OK
    assert grid == 2 * sms
    all_rows = spans.cpu().numpy()
    assert (all_rows[grid:] == 0).all()  # one row per launched CTA, no more
    sp = all_rows[:grid]
    smid, t0, t1 = sp[:, 0], sp[:, 1], sp[:, 2]
    assert (t1 > t0).all()
    per_sm = Counter(smid.tolist())
    assert len(per_sm) == sms and set(per_sm.values()) == {2}
    for s in per_sm:
        a, b = np.nonzero(smid == s)[0]
        assert max(t0[a], t0[b]) < min(t1[a], t1[b]), f"SM {s}: the two CTAs did not run at the same time"
    o2, l2 = vb.attention(q, k, v, None, CROSS, 0)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_cross_attention_is_deterministic():
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in wl.draw_qkv(1, 8, 20000, 512, 128, seed=42, recipe="rms_qk"))
    o1, l1 = vb.attention(q, k, v, None, CROSS, 0)
    o2, l2 = vb.attention(q, k, v, None, CROSS, 0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_parity_other_scales():
    q, k, v = wl.draw_qkv(1, 2, 400, 400, 128, seed=3, recipe="iid")
    for scale in (0.02, 0.2):
        compare_all_rows(q, k, v, scale, FULL, 0, f"scale {scale}")


@pytest.mark.parametrize("mask,chunk", [(FULL, 0), (BC, 500)])
def test_running_max_jumps_force_rescaling(mask, chunk):
    """Later key tiles carry much larger logits, so the running row max grows
    far past the lazy-rescale threshold mid-sequence (and once more inside a
    tile that is only partly allowed)."""
    B, H, S, D = 1, 2, 1000, 128
    q, k, v = wl.draw_qkv(B, H, S, S, D, seed=21, recipe="rms_qk")
    k = k.float()
    k[:, 300:428] *= 6.0   # keys across the tile 2/3 boundary: row max ~4 -> ~21 (log2 units)
    k[:, 700:760] *= 12.0  # inside tile 5: row max -> ~40
    compare_all_rows(q, k.to(torch.bfloat16), v, 1 / math.sqrt(D), mask, chunk, f"rescale m{mask}")
    # descending: the largest logits come first, later tiles never rescale
    k2 = wl.draw_qkv(B, H, S, S, D, seed=22, recipe="rms_qk")[1].float()
    k2[:, :128] *= 10.0
    compare_all_rows(q, k2.to(torch.bfloat16), v, 1 / math.sqrt(D), mask, chunk, f"no-rescale m{mask}")


def test_constant_values_and_zero_queries():
    B, H, S, D = 1, 2, 700, 128
    q, k, _ = wl.draw_qkv(B, H, S, S, D, seed=11, recipe="rms_qk")
    const = torch.randn(1, 1, H, D).to(torch.bfloat16)
    v = const.expand(B, S, H, D).contiguous()
    for mask, chunk in [(FULL, 0), (BC, 300)]:
        o, _ = run_gpu(q, k, v, 1 / math.sqrt(D), mask, chunk)
        expect = np.broadcast_to(const.double().numpy(), o.shape)
        assert np.max(np.abs(o - expect)) <= 1e-2 * max(1.0, float(np.abs(expect).max()))
    # Q = 0: every row is the mean of its allowed value rows, LSE = ln |A(i)|
    _, _, v = wl.draw_qkv(B, H, S, S, D, seed=12, recipe="iid")
    qz = torch.zeros_like(q)
    o, lse = run_gpu(qz, k, v, 1 / math.sqrt(D), BC, 300)
    vv = v.double().numpy()
    for i in (0, 299, 300, 599, 600, 699):
        n = min(S, (i // 300 + 1) * 300)
        np.testing.assert_allclose(o[0, i], round_bf16(vv[0, :n].mean(axis=0)), atol=2e-3)
        np.testing.assert_allclose(lse[0, :, i], math.log(n), rtol=1e-3)


def test_joint_permutation_of_keys_and_values():
    q, k, v = wl.draw_qkv(1, 2, 500, 900, 128, seed=13, recipe="rms_qk")
    perm = torch.randperm(900, generator=torch.Generator().manual_seed(0))
    o1, l1 = run_gpu(q, k, v, 1 / math.sqrt(128), CROSS)
    o2, l2 = run_gpu(q, k[:, perm].contiguous(), v[:, perm].contiguous(), 1 / math.sqrt(128), CROSS)
    assert np.max(np.abs(o1 - o2)) <= 1e-2 and np.mean(np.abs(o1 - o2)) <= 1e-3
    assert np.max(np.abs(l1 - l2)) <= 1e-3 * np.max(np.abs(l1))


def test_lse_merges_two_key_halves():
    q, k, v = wl.draw_qkv(1, 3, 640, 1000, 128, seed=14, recipe="rms_qk")
    s = 1 / math.sqrt(128)
    o, l = run_gpu(q, k, v, s, CROSS)
    o1, l1 = run_gpu(q, k[:, :384].contiguous(), v[:, :384].contiguous(), s, CROSS)
    o2, l2 = run_gpu(q, k[:, 384:].contiguous(), v[:, 384:].contiguous(), s, CROSS)
    lm = np.logaddexp(l1, l2)
    w1 = np.exp(l1 - lm).transpose(0, 2, 1)[..., None]
    w2 = np.exp(l2 - lm).transpose(0, 2, 1)[..., None]
    merged = w1 * o1 + w2 * o2
    assert np.max(np.abs(merged - o)) <= 1e-2
    assert np.max(np.abs(lm - l)) <= 1e-3 * np.max(np.abs(l))


def test_bitwise_deterministic():
    dev = torch.device("cuda:0")
    for mask, chunk in [(FULL, 0), (BC, 700)]:
        q, k, v = (t.to(dev) for t in wl.draw_qkv(1, 4, 2000, 2000, 128, seed=15, recipe="rms_qk"))
        o1, l1 = vb.attention(q, k, v, None, mask, chunk)
        o2, l2 = vb.attention(q, k, v, None, mask, chunk)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("mask,Skv", [(FULL, 300), (CROSS, 77)])
def test_writes_stay_inside_the_output_buffers(mask, Skv):
    # the cross kernel stores O with TMA boxes of 32 rows: Sq = 300 ends inside one
    dev = torch.device("cuda:0")
    B, H, Sq, D = 1, 2, 300, 128
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, Sq, Skv, D, seed=16))
    n_o, n_l, guard = B * Sq * H * D, B * H * Sq, 4096
    o_buf = torch.full((n_o + guard,), 7.0, dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((n_l + guard,), 7.0, dtype=torch.float32, device=dev)
    vb.vdit_attn_fwd(q, k, v, o_buf.data_ptr(), l_buf.data_ptr(), B, H, Sq, Skv, D, 1 / math.sqrt(D),
                     mask, 0)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(l_buf[n_l:] == 7.0)
    assert torch.isfinite(o_buf[:n_o].float()).all() and torch.isfinite(l_buf[:n_l]).all()


def test_lse_is_optional():
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in wl.draw_qkv(1, 2, 300, 300, 128, seed=17))
    o1 = vb.attention(q, k, v, None, FULL, 0, return_lse=False)
    o2, _ = vb.attention(q, k, v, None, FULL, 0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


# 512 rows per head (every head), including the first and last rows and the
# rows on both sides of tile and chunk boundaries; each row is computed by the
# oracle exactly, against all of its allowed keys
LARGE = [
    ("wan21_1p3b_480p", 0, 512),
    ("wan22_720p_16x16", 0, 512),
    ("wan21_14b_720p", 0, 512),
    ("wan21_14b_720p", 1, 512),
    ("block_causal_7x4680", 0, 512),
]


@pytest.mark.parametrize("name,call_idx,per_head", LARGE)
def test_parity_full_size_workloads_sampled(name, call_idx, per_head):
    """Full-size workloads in the benchmark's launch configuration, sampled rows."""
    w = wl.WORKLOADS[name]
    call = w.calls[call_idx]
    inp = wl.workload_inputs(name)
    q = inp["q"]
    k, v = (inp["k_text"], inp["v_text"]) if call.mask_kind == CROSS else (inp["k"], inp["v"])
    o_g, l_g = run_gpu(q, k, v, call.scale, call.mask_kind, call.chunk_tokens)
    rows = wl.sample_rows(call.B, call.H, call.Sq, per_head, seed=100 + w.index, chunk_tokens=call.chunk_tokens)
    o_r, l_r = oracle_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), call.scale,
                                call.mask_kind, call.chunk_tokens, rows=rows)
    o_s = o_g[rows[:, 0], rows[:, 2], rows[:, 1]]
    l_s = l_g[rows[:, 0], rows[:, 1], rows[:, 2]]
    groups = [np.nonzero((rows[:, 0] == b) & (rows[:, 1] == h))[0] for b in range(call.B) for h in range(call.H)]
    res = check_parity(o_s, o_r, l_s, l_r, groups, f"{name}/{call.name}")
    assert res["ok"], res
