"""The 8-bit path (E4M3 + V-Smooth + ExpCast-FP8) on the GPU against its oracle.

The preprocessing writes integer codes and fp32 scales that the oracle
computes with the same fp32 operations: those must match bit for bit.

The attention is checked twice.  Against the plain statement of ExpCast
(oracle.fp8_oracle.attention_fp8_plain: every probability byte against its
row's true maximum, no tiles, no running reference), under the bars derived
in tests/helpers.py from the byte map's own log error -- the independent
check.  And against attention_fp8, which walks the keys in the kernel's
schedule, under the bf16 path's parity bars -- a tighter check that the
kernel's bytes are the ones its schedule defines (they can differ by one
code where the tensor core's fp32 scores round a tie differently from the
oracle's float64 ones).
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as exact_attention
from oracle import fp8_oracle as f8
from tests.helpers import check_expcast_parity, check_parity
from video_diffusion_transformer_attention_b200 import binding as vb
from video_diffusion_transformer_attention_b200 import workloads as wl
from video_diffusion_transformer_attention_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib(cuda_device):
    build()
    return vb.lib()


def _quantize(q, k, v):
    dev = torch.device("cuda:0")
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    st, parts, total = vb.vdit_fp8_layout(B, H, Sq, Skv, D)
    assert st == vb.VDIT_OK
    ws = torch.empty(total, dtype=torch.uint8, device=dev)
    vb.vdit_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), B, H, Sq, Skv, D, ws, total)
    torch.cuda.synchronize()
    return ws.cpu().numpy(), parts, total


def _part(ws, parts, name, dtype, count):
    o = parts[name]
    return np.frombuffer(ws[o:o + count * np.dtype(dtype).itemsize].tobytes(), dtype=dtype)


@pytest.mark.parametrize("B,H,Sq,Skv", [(1, 2, 256, 256), (2, 3, 300, 333), (1, 1, 129, 77)])
def test_quantisation_is_bit_exact(B, H, Sq, Skv):
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=91 + Sq, recipe="rms_qk_vout")
    ws, parts, _ = _quantize(q, k, v)
    qc, qs = f8.quantize_qk(wl.bf16_bits(q))
    kc, ks = f8.quantize_qk(wl.bf16_bits(k))
    vs = f8.vsmooth(wl.bf16_bits(v))
    nqb, nkb = -(-Sq // 128), -(-Skv // 128)
    assert np.array_equal(_part(ws, parts, "q", np.uint8, qc.size).reshape(qc.shape), qc)
    assert np.array_equal(_part(ws, parts, "k", np.uint8, kc.size).reshape(kc.shape), kc)
    assert np.array_equal(_part(ws, parts, "q_scale", np.float32, B * H * nqb).reshape(qs.shape), qs)
    assert np.array_equal(_part(ws, parts, "k_scale", np.float32, B * H * nkb).reshape(ks.shape), ks)
    assert np.array_equal(_part(ws, parts, "v_scale", np.float32, B * H * 128).reshape(B, H, 128), vs["scale"])
    assert np.array_equal(_part(ws, parts, "mu", np.float32, B * H * nkb * 128).reshape(B, H, nkb, 128), vs["mu"])
    vt = _part(ws, parts, "vt", np.uint8, B * H * nkb * 128 * 128).reshape(B, H, nkb, 128, 128)
    want = np.zeros((B, H, nkb * 128, 128), np.uint8)
    want[:, :, :Skv] = vs["codes"].transpose(0, 2, 1, 3)
    assert np.array_equal(vt.transpose(0, 1, 2, 4, 3).reshape(B, H, nkb * 128, 128), want)
    # restore tiles: rows 0, 1, 2 = mu'_hi, mu'_hi, mu'_lo at their 128B-swizzled places, zeros elsewhere
    img = _part(ws, parts, "mu_img", np.uint8, B * H * nkb * 4096).reshape(B, H, nkb, 4096)
    d = np.arange(128)
    half, c = d // 64, d % 64
    expect = np.zeros((B, H, nkb, 2048), np.uint16)
    for row, src in ((0, vs["mu_hi"]), (1, vs["mu_hi"]), (2, vs["mu_lo"])):
        pos = (half * 2048 + row * 128 + (((c >> 3) ^ row) << 4) + (c & 7) * 2) // 2
        expect[:, :, :, pos] = src
    assert np.array_equal(img.view(np.uint16), expect)


def _run_fp8(q, k, v, mask, chunk, scale):
    dev = torch.device("cuda:0")
    o, lse, _ = vb.attention_fp8(q.to(dev), k.to(dev), v.to(dev), scale, mask, chunk)
    st, word = vb.vdit_get_device_status()
    assert st == vb.VDIT_OK, f"device status {vb.vdit_status_string(st)} word={word:#x}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _flat(o, lse, B, H):
    og = np.concatenate([o[b, :, h] for b in range(B) for h in range(H)])
    lg = np.concatenate([lse[b, h] for b in range(B) for h in range(H)])
    return og, lg


CASES = [  # B, H, Sq, Skv, mask, chunk, recipe
    (1, 2, 256, 256, vb.VDIT_MASK_FULL, 0, "rms_qk"),
    (1, 2, 1000, 1000, vb.VDIT_MASK_FULL, 0, "rms_qk_vout"),
    (2, 3, 300, 333, vb.VDIT_MASK_FULL, 0, "iid"),
    (1, 2, 700, 77, vb.VDIT_MASK_CROSS, 0, "rms_qk"),
    (1, 2, 1000, 1000, vb.VDIT_MASK_BLOCK_CAUSAL, 300, "rms_qk"),
    (1, 1, 129, 129, vb.VDIT_MASK_BLOCK_CAUSAL, 1, "iid"),
]


@pytest.mark.parametrize("B,H,Sq,Skv,mask,chunk,recipe", CASES)
def test_fp8_attention_matches_its_oracle(B, H, Sq, Skv, mask, chunk, recipe):
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=92 + Sq + Skv, recipe=recipe)
    scale = 1 / math.sqrt(128)
    o, lse = _run_fp8(q, k, v, mask, chunk, scale)
    o_r, l_r = f8.attention_fp8(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, mask, chunk)
    og, lg = _flat(o, lse, B, H)
    orr, lr = _flat(o_r, l_r, B, H)
    groups = [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)]
    res = check_parity(og, orr, lg, lr, groups, f"fp8 {B}x{H}x{Sq}x{Skv} m{mask}",
                       excess_bar=None)  # 8-bit arithmetic: its ExpCast bytes may differ by one code at ties
    assert res["ok"], res


@pytest.mark.parametrize("B,H,Sq,Skv,mask,chunk,recipe", CASES)
def test_fp8_attention_matches_the_plain_expcast_statement(B, H, Sq, Skv, mask, chunk, recipe):
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=92 + Sq + Skv, recipe=recipe)
    scale = 1 / math.sqrt(128)
    o, lse = _run_fp8(q, k, v, mask, chunk, scale)
    o_p, l_p, s_o, s_l = f8.attention_fp8_plain(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, mask,
                                                 chunk, spread=True)
    og, lg = _flat(o, lse, B, H)
    op, lp = _flat(o_p, l_p, B, H)
    so, sl = _flat(s_o, s_l, B, H)
    groups = [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)]
    res = check_expcast_parity(og, op, lg, lp, so, sl, groups, f"fp8 plain {B}x{H}x{Sq}x{Skv} m{mask}")
    assert res["ok"], res


def test_fp8_attention_with_a_wide_logit_span_takes_the_exact_clamp_and_matches():
    # Q and K x30: |logit| reaches the thousands of code units, beyond what the
    # 16-bit clamp may handle, so every warp runs the float-clamp loop
    B, H, S = 1, 2, 600
    q, k, v = wl.draw_qkv(B, H, S, S, 128, seed=96, recipe="iid")
    q = (q.float() * 30).to(torch.bfloat16)
    k = (k.float() * 30).to(torch.bfloat16)
    scale = 1 / math.sqrt(128)
    o, lse = _run_fp8(q, k, v, vb.VDIT_MASK_FULL, 0, scale)
    o_r, l_r = f8.attention_fp8(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale)
    og, lg = _flat(o, lse, B, H)
    orr, lr = _flat(o_r, l_r, B, H)
    res = check_parity(og, orr, lg, lr, [np.arange(i * S, (i + 1) * S) for i in range(B * H)], "fp8 wide span",
                       excess_bar=None)
    assert res["ok"], res


def test_fp8_attention_is_close_to_exact_attention():
    B, H, S = 1, 2, 1000
    q, k, v = wl.draw_qkv(B, H, S, S, 128, seed=93, recipe="rms_qk_vout")
    scale = 1 / math.sqrt(128)
    o, lse = _run_fp8(q, k, v, vb.VDIT_MASK_FULL, 0, scale)
    o_x, l_x = exact_attention(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale)
    rel = np.sqrt(((o - o_x) ** 2).mean()) / np.sqrt((o_x ** 2).mean())
    assert rel < 0.10, rel
    assert (np.abs(lse - l_x) / np.maximum(np.abs(l_x), 1)).max() < 0.03


def test_two_step_api_equals_the_combined_entry_and_is_deterministic():
    dev = torch.device("cuda:0")
    B, H, S = 1, 3, 777
    q, k, v = (t.to(dev) for t in wl.draw_qkv(B, H, S, S, 128, seed=94, recipe="rms_qk"))
    o1, l1, ws = vb.attention_fp8(q, k, v, None, vb.VDIT_MASK_BLOCK_CAUSAL, 256)
    o2, l2, _ = vb.attention_fp8(q, k, v, None, vb.VDIT_MASK_BLOCK_CAUSAL, 256, workspace=ws)
    ws2 = torch.empty_like(ws)
    vb.vdit_fp8_quantize(q, k, v, B, H, S, S, 128, ws2, ws2.numel())
    o3, l3 = torch.empty_like(o1), torch.empty_like(l1)
    vb.vdit_attn_fwd_fp8_quantized(o3, l3, B, H, S, S, 128, 1 / math.sqrt(128), vb.VDIT_MASK_BLOCK_CAUSAL, 256,
                                   ws2, ws2.numel())
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_fp8_attention_sampled_rows_at_a_wan_shape():
    name = "wan22_720p_16x16"
    w = wl.WORKLOADS[name]
    call = w.calls[0]
    inp = wl.workload_inputs(name)
    q, k, v = inp["q"], inp["k"], inp["v"]
    o, lse = _run_fp8(q, k, v, call.mask_kind, call.chunk_tokens, call.scale)
    rows = wl.sample_rows(call.B, call.H, call.Sq, 8, seed=95)
    quant = (f8.quantize_qk(wl.bf16_bits(q)), f8.quantize_qk(wl.bf16_bits(k)), f8.vsmooth(wl.bf16_bits(v)))
    o_r, l_r = f8.attention_fp8(None, None, None, call.scale, call.mask_kind, call.chunk_tokens, rows=rows,
                                quantized=quant)
    og = np.stack([o[b, i, h] for b, h, i in rows])
    lg = np.array([lse[b, h, i] for b, h, i in rows])
    res = check_parity(og, o_r, lg, l_r, None, f"fp8 {name} sampled", excess_bar=None)
    assert res["ok"], res
    # the same rows against the plain ExpCast statement
    o_p, l_p, s_o, s_l = f8.attention_fp8_plain(None, None, None, call.scale, call.mask_kind, call.chunk_tokens,
                                                 rows=rows, quantized=quant, spread=True)
    groups = [np.nonzero(rows[:, 1] == h)[0] for h in range(call.H)]
    res = check_expcast_parity(og, o_p, lg, l_p, s_o, s_l, groups, f"fp8 plain {name} sampled")
    assert res["ok"], res


def test_fp8_cross_attention_sampled_rows_at_the_bench_shape():
    # Sq = 75,600, H = 40, Skv = 512 text tokens: the persistent cross kernel
    # takes ~80 query tiles per CTA, so its barrier phases run across items
    name = "wan21_14b_720p"
    call = wl.WORKLOADS[name].calls[1]
    inp = wl.workload_inputs(name)
    q, k, v = inp["q"], inp["k_text"], inp["v_text"]
    o, lse = _run_fp8(q, k, v, call.mask_kind, call.chunk_tokens, call.scale)
    rows = wl.sample_rows(call.B, call.H, call.Sq, 8, seed=97)
    quant = (f8.quantize_qk(wl.bf16_bits(q)), f8.quantize_qk(wl.bf16_bits(k)), f8.vsmooth(wl.bf16_bits(v)))
    o_r, l_r = f8.attention_fp8(None, None, None, call.scale, call.mask_kind, call.chunk_tokens, rows=rows,
                                quantized=quant)
    og = np.stack([o[b, i, h] for b, h, i in rows])
    lg = np.array([lse[b, h, i] for b, h, i in rows])
    res = check_parity(og, o_r, lg, l_r, None, f"fp8 {name} cross sampled", excess_bar=None)
    assert res["ok"], res
    o_p, l_p, s_o, s_l = f8.attention_fp8_plain(None, None, None, call.scale, call.mask_kind, call.chunk_tokens,
                                                 rows=rows, quantized=quant, spread=True)
    groups = [np.nonzero(rows[:, 1] == h)[0] for h in range(call.H)]
    res = check_expcast_parity(og, o_p, lg, l_p, s_o, s_l, groups, f"fp8 plain {name} cross sampled")
    assert res["ok"], res


def test_fp8_cross_attention_all_rows_several_items_per_cta():
    # 600 query tiles over 296 CTAs: every CTA runs two or three items
    B, H, Sq, Skv = 1, 4, 128 * 150 - 37, 300
    q, k, v = wl.draw_qkv(B, H, Sq, Skv, 128, seed=98, recipe="rms_qk")
    scale = 1 / math.sqrt(128)
    o, lse = _run_fp8(q, k, v, vb.VDIT_MASK_CROSS, 0, scale)
    o_r, l_r = f8.attention_fp8(wl.bf16_bits(q), wl.bf16_bits(k), wl.bf16_bits(v), scale, vb.VDIT_MASK_CROSS, 0)
    og, lg = _flat(o, lse, B, H)
    orr, lr = _flat(o_r, l_r, B, H)
    res = check_parity(og, orr, lg, lr, [np.arange(i * Sq, (i + 1) * Sq) for i in range(B * H)],
                       "fp8 cross, several items per CTA", excess_bar=None)
    assert res["ok"], res
