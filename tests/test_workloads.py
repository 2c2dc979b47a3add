"""Workload shapes, input recipe and the FLOP counter, pinned to the pages."""
import math
import os

import numpy as np
import torch

from video_diffusion_transformer_attention_b200 import flops, workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=")
            vals[k] = float(v)
    return vals


def test_token_counts_match_the_pages():
    g = read_golden("sudonull_flop_breakdown.txt")
    assert g["tokens_temporal"] * g["tokens_spatial"] == g["tokens_total"]
    w = wl.WORKLOADS["wan21_14b_720p"].calls[0]
    assert w.Sq == g["tokens_total"] and w.H * w.D == g["d_model"]
    assert wl.WORKLOADS["wan22_720p_16x16"].calls[0].Sq == g["wan22_16x16_tokens"]
    c = read_golden("waveforcing_chunks.txt")
    bc = wl.WORKLOADS["block_causal_7x4680"].calls[0]
    assert bc.chunk_tokens == c["frames_per_chunk"] * c["tokens_per_frame"]
    assert bc.Sq == c["latent_frames"] * c["tokens_per_frame"]
    assert c["latent_frames"] % c["frames_per_chunk"] == 0


def test_flop_counter_reproduces_the_page_breakdown():
    g = read_golden("sudonull_flop_breakdown.txt")
    S, d, dff = g["tokens_total"], g["d_model"], g["d_ff"]
    core = flops.attn_flops(wl.WORKLOADS["wan21_14b_720p"].calls[0])
    assert core == 4 * S * S * d  # 117.05 TFLOP
    assert abs(core / 1e12 - 117.05) < 0.01
    # the page's self-attention figure adds the Q/K/V/O projections (8 S d^2)
    self_attn = core + 8 * S * d * d
    assert abs(self_attn / 1e12 - g["self_attention_tflop_per_layer"]) / g["self_attention_tflop_per_layer"] < 0.005
    ffn = 4 * S * d * dff
    assert abs(ffn / 1e12 - g["ffn_tflop_per_layer"]) < 0.05
    # self-attention share of the page's layer total
    assert abs(100 * self_attn / 1e12 / g["layer_total_tflop"] - g["self_attention_share_percent"]) < 1.0
    cross_core = flops.attn_flops(wl.WORKLOADS["wan21_14b_720p"].calls[1])
    assert abs(cross_core / 1e12 - 0.7927) < 1e-3


def test_block_causal_pair_count_brute_force():
    for S, c in [(17, 5), (32, 8), (10, 3), (9, 20)]:
        brute = sum(1 for i in range(S) for j in range(S) if j // c <= i // c)
        assert flops.allowed_pairs(S, S, wl.MASK_BLOCK_CAUSAL, c) == brute
    bc = wl.WORKLOADS["block_causal_7x4680"].calls[0]
    # 7 equal chunks: 28 of the 49 chunk pairs are allowed
    assert flops.allowed_pairs(bc.Sq, bc.Skv, bc.mask_kind, bc.chunk_tokens) * 49 == 28 * bc.Sq * bc.Skv


def test_draws_are_seeded_and_follow_the_recipe():
    q1, k1, v1 = wl.draw_qkv(1, 3, 64, 64, 128, 7, "rms_qk_vout")
    q2, k2, v2 = wl.draw_qkv(1, 3, 64, 64, 128, 7, "rms_qk_vout")
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    assert q1.dtype == torch.bfloat16 and q1.shape == (1, 64, 3, 128)
    ms = q1.float().pow(2).mean(-1)
    assert torch.allclose(ms, torch.ones_like(ms), atol=2e-2)
    # three channels per head carry the x8 gain: their RMS stands out
    rms = v1.float().pow(2).mean(dim=(0, 1)).sqrt()  # [H, D]
    for h in range(3):
        big = (rms[h] > 4).nonzero().flatten()
        assert len(big) == wl.OUTLIER_CHANNELS
    q3, _, _ = wl.draw_qkv(1, 3, 64, 64, 128, 8, "rms_qk")
    assert not torch.equal(q1, q3)


def test_sample_rows_cover_boundaries():
    rows = wl.sample_rows(1, 2, 1000, 40, 0, chunk_tokens=300)
    for h in range(2):
        r = set(rows[rows[:, 1] == h][:, 2].tolist())
        assert {0, 999, 127, 128, 299, 300, 599, 600}.issubset(r)
        assert len(r) >= 40
    assert np.all((rows[:, 2] >= 0) & (rows[:, 2] < 1000))


def test_scale_is_inverse_sqrt_head_dim():
    assert math.isclose(wl.WORKLOADS["pr1_s1024"].calls[0].scale, 1 / math.sqrt(128))
