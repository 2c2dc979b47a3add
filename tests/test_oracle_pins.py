"""Pins for the fp64 oracle: each checks it against something other than itself.

Closed forms, a library routine (torch's float64 scaled_dot_product_attention
and logsumexp on the CPU), exact special cases of the block-causal rule, and
the invariants the pages state: non-causal attention is unchanged when keys and
values are permuted together, and a constant added to every value row comes
back out unchanged because softmax rows sum to one ("VC-Attention"
(aikraft.ru), section 02 "V-Smooth", the Group and Restore steps).

The pins are chosen so that a plausible slip in the oracle -- a dropped scale,
a wrong sign, a transposed operand, a layout or index mix-up, log2 instead of
ln, an off-by-one in the chunk rule -- fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import MASK_BLOCK_CAUSAL, MASK_CROSS, MASK_FULL, attention
from tests.helpers import bits_to_float, to_bf16_bits


def rand_bits(rng, shape, std=1.0):
    return to_bf16_bits(rng.standard_normal(shape) * std)


def sdpa_reference(qb, kb, vb, scale, mask=None):
    """torch float64 attention + logsumexp, [B,S,H,D] in, ([B,Sq,H,D], [B,H,Sq]) out."""
    q = torch.from_numpy(bits_to_float(qb)).permute(0, 2, 1, 3)
    k = torch.from_numpy(bits_to_float(kb)).permute(0, 2, 1, 3)
    v = torch.from_numpy(bits_to_float(vb)).permute(0, 2, 1, 3)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask, scale=scale)
    logits = (q @ k.transpose(-1, -2)) * scale
    if mask is not None:
        logits = logits.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def block_causal_mask(S, c):
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    return (j // c) <= (i // c)


@pytest.mark.parametrize("B,H,Sq,Skv,D", [(2, 3, 37, 37, 16), (1, 2, 19, 53, 32), (2, 1, 5, 7, 8)])
def test_full_matches_torch_sdpa_fp64(B, H, Sq, Skv, D):
    rng = np.random.default_rng(1)
    qb, kb, vb = (rand_bits(rng, (B, Sq, H, D)), rand_bits(rng, (B, Skv, H, D)),
                  rand_bits(rng, (B, Skv, H, D)))
    scale = 1.0 / math.sqrt(D)
    for mk in (MASK_FULL, MASK_CROSS):
        o, lse = attention(qb, kb, vb, scale, mk)
        o_ref, lse_ref = sdpa_reference(qb, kb, vb, scale)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("S,c", [(40, 7), (33, 11), (16, 16), (9, 4)])
def test_block_causal_matches_torch_sdpa_masked(S, c):
    rng = np.random.default_rng(2)
    B, H, D = 2, 2, 16
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    scale = 0.3
    o, lse = attention(qb, kb, vb, scale, MASK_BLOCK_CAUSAL, c)
    o_ref, lse_ref = sdpa_reference(qb, kb, vb, scale, block_causal_mask(S, c))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_block_causal_chunk_one_is_token_causal():
    rng = np.random.default_rng(3)
    B, H, S, D = 1, 3, 23, 16
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    o, lse = attention(qb, kb, vb, 0.25, MASK_BLOCK_CAUSAL, 1)
    q = torch.from_numpy(bits_to_float(qb)).permute(0, 2, 1, 3)
    k = torch.from_numpy(bits_to_float(kb)).permute(0, 2, 1, 3)
    v = torch.from_numpy(bits_to_float(vb)).permute(0, 2, 1, 3)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o_ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, is_causal=True, scale=0.25)
    np.testing.assert_allclose(o, o_ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_block_causal_chunk_covering_sequence_is_full():
    rng = np.random.default_rng(4)
    B, H, S, D = 1, 2, 31, 16
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    o_full, l_full = attention(qb, kb, vb, 0.2, MASK_FULL)
    for c in (S, S + 5, 1000):
        o, l = attention(qb, kb, vb, 0.2, MASK_BLOCK_CAUSAL, c)
        np.testing.assert_array_equal(o, o_full)
        np.testing.assert_array_equal(l, l_full)


def test_block_causal_rows_equal_full_over_truncated_keys():
    """Rows of chunk m see exactly keys [0, (m+1)c): compare with FULL on K[:(m+1)c]."""
    rng = np.random.default_rng(5)
    B, H, S, D, c = 1, 2, 26, 16, 6
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    o, lse = attention(qb, kb, vb, 0.2, MASK_BLOCK_CAUSAL, c)
    for m in range((S + c - 1) // c):
        end = min(S, (m + 1) * c)
        rows = slice(m * c, min(S, (m + 1) * c))
        o_t, l_t = attention(qb[:, rows], kb[:, :end], vb[:, :end], 0.2, MASK_CROSS)
        np.testing.assert_array_equal(o[:, rows], o_t)
        np.testing.assert_array_equal(lse[:, :, rows], l_t)


@pytest.mark.parametrize("mk,c", [(MASK_FULL, 0), (MASK_BLOCK_CAUSAL, 5), (MASK_CROSS, 0)])
def test_constant_values_give_that_constant(mk, c):
    rng = np.random.default_rng(6)
    B, H, S, D = 2, 2, 17, 16
    qb, kb = rand_bits(rng, (B, S, H, D), 2.0), rand_bits(rng, (B, S, H, D), 2.0)
    const = rand_bits(rng, (1, 1, H, D))
    vb = np.broadcast_to(const, (B, S, H, D)).copy()
    o, _ = attention(qb, kb, vb, 0.5, mk, c)
    expect = np.broadcast_to(bits_to_float(const), o.shape)
    np.testing.assert_allclose(o, expect, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("mk,c", [(MASK_FULL, 0), (MASK_BLOCK_CAUSAL, 4)])
def test_zero_query_gives_mean_of_allowed_values(mk, c):
    rng = np.random.default_rng(7)
    B, H, S, D = 1, 3, 18, 8
    qb = np.zeros((B, S, H, D), np.uint16)  # bf16 +0.0
    kb, vb = rand_bits(rng, (B, S, H, D)), rand_bits(rng, (B, S, H, D))
    o, lse = attention(qb, kb, vb, 0.7, mk, c)
    v = bits_to_float(vb)
    for i in range(S):
        n = S if mk == MASK_FULL else min(S, (i // c + 1) * c)
        np.testing.assert_allclose(o[:, i], v[:, :n].mean(axis=1), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value_row():
    rng = np.random.default_rng(8)
    B, H, S, D = 1, 1, 12, 16
    q = np.zeros((B, S, H, D))
    k = rng.standard_normal((B, S, H, D)) * 0.05
    q[0, 3, 0, 0] = 8.0
    k[0, 9, 0, :] = 0.0
    k[0, 9, 0, 0] = 64.0  # logit 8*64*scale = 128, the others |.| < 8
    qb, kb, vb = to_bf16_bits(q), to_bf16_bits(k), rand_bits(rng, (B, S, H, D))
    o, lse = attention(qb, kb, vb, 0.25, MASK_FULL)
    np.testing.assert_allclose(o[0, 3, 0], bits_to_float(vb)[0, 9, 0], rtol=1e-20, atol=1e-20)
    assert abs(lse[0, 0, 3] - 128.0) < 1e-20 + 128.0 * 1e-16


def test_two_keys_logistic_closed_form():
    """Skv = 2: O = s(l0-l1) v0 + s(l1-l0) v1, LSE = l0 + ln(1 + e^(l1-l0))."""
    rng = np.random.default_rng(9)
    D = 8
    qb = rand_bits(rng, (1, 1, 1, D))
    kb = rand_bits(rng, (1, 2, 1, D))
    vb = rand_bits(rng, (1, 2, 1, D))
    q, k, v = bits_to_float(qb)[0, 0, 0], bits_to_float(kb)[0, :, 0], bits_to_float(vb)[0, :, 0]
    # bf16 x bf16 products and their 8-term sums are exact in binary64
    l0 = 0.5 * sum(float(q[d]) * float(k[0, d]) for d in range(D))
    l1 = 0.5 * sum(float(q[d]) * float(k[1, d]) for d in range(D))
    w0 = 1.0 / (1.0 + math.exp(l1 - l0))
    expect_o = w0 * v[0] + (1.0 - w0) * v[1]
    expect_lse = l0 + math.log1p(math.exp(l1 - l0))
    o, lse = attention(qb, kb, vb, 0.5, MASK_FULL)
    np.testing.assert_allclose(o[0, 0, 0], expect_o, rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - expect_lse) < 1e-14


def test_joint_key_value_permutation_invariance():
    rng = np.random.default_rng(10)
    B, H, S, D, c = 1, 2, 30, 16, 10
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    o, lse = attention(qb, kb, vb, 0.3, MASK_FULL)
    perm = rng.permutation(S)
    o_p, lse_p = attention(qb, kb[:, perm], vb[:, perm], 0.3, MASK_FULL)
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse_p, lse, rtol=0, atol=1e-13)
    # block-causal: permuting within each chunk keeps every allowed set
    perm_bc = np.concatenate([s + rng.permutation(min(c, S - s)) for s in range(0, S, c)])
    o_bc, l_bc = attention(qb, kb, vb, 0.3, MASK_BLOCK_CAUSAL, c)
    o_bcp, l_bcp = attention(qb, kb[:, perm_bc], vb[:, perm_bc], 0.3, MASK_BLOCK_CAUSAL, c)
    np.testing.assert_allclose(o_bcp, o_bc, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_bcp, l_bc, rtol=0, atol=1e-13)


def test_shift_equivariance_in_values():
    """attn(Q, K, V + 1 c^T) = attn(Q, K, V) + c (rows of the softmax sum to one)."""
    rng = np.random.default_rng(11)
    B, H, S, D = 1, 2, 21, 16
    qb, kb = rand_bits(rng, (B, S, H, D)), rand_bits(rng, (B, S, H, D))
    v = np.round(rng.standard_normal((B, S, H, D)) * 4) / 4  # exact in bf16
    shift = np.round(rng.standard_normal((1, 1, H, D)) * 4) / 4
    o, _ = attention(qb, kb, to_bf16_bits(v), 0.25, MASK_BLOCK_CAUSAL, 4)
    o_s, _ = attention(qb, kb, to_bf16_bits(v + shift), 0.25, MASK_BLOCK_CAUSAL, 4)
    np.testing.assert_allclose(o_s, o + shift, rtol=0, atol=1e-13)


def test_lse_merge_of_two_key_halves_equals_full():
    rng = np.random.default_rng(12)
    B, H, Sq, Skv, D, split = 1, 2, 9, 40, 16, 17
    qb, kb, vb = rand_bits(rng, (B, Sq, H, D)), rand_bits(rng, (B, Skv, H, D)), rand_bits(rng, (B, Skv, H, D))
    o, lse = attention(qb, kb, vb, 0.25, MASK_CROSS)
    o1, l1 = attention(qb, kb[:, :split], vb[:, :split], 0.25, MASK_CROSS)
    o2, l2 = attention(qb, kb[:, split:], vb[:, split:], 0.25, MASK_CROSS)
    lm = np.logaddexp(l1, l2)
    w1 = np.exp(l1 - lm).transpose(0, 2, 1)[..., None]
    w2 = np.exp(l2 - lm).transpose(0, 2, 1)[..., None]
    np.testing.assert_allclose(w1 * o1 + w2 * o2, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lm, lse, rtol=0, atol=1e-13)


def test_row_selection_matches_full_run():
    rng = np.random.default_rng(13)
    B, H, S, D = 2, 3, 25, 16
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    o, lse = attention(qb, kb, vb, 0.25, MASK_BLOCK_CAUSAL, 6)
    rows = np.array([(1, 2, 24), (0, 0, 0), (1, 0, 6), (0, 1, 5)])
    o_s, l_s = attention(qb, kb, vb, 0.25, MASK_BLOCK_CAUSAL, 6, rows=rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o_s[n], o[b, i, h])
        assert l_s[n] == lse[b, h, i]


def test_no_keys_gives_zero_output_and_minus_inf_lse():
    qb = np.zeros((1, 3, 1, 8), np.uint16)
    kb = np.zeros((1, 0, 1, 8), np.uint16)
    o, lse = attention(qb, kb, kb, 0.5, MASK_CROSS)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


def test_oracle_rejects_bad_arguments():
    qb = np.zeros((1, 4, 1, 8), np.uint16)
    with pytest.raises(ValueError):
        attention(qb, qb, qb, 0.5, 7)
    with pytest.raises(ValueError):
        attention(qb, qb, qb, 0.5, MASK_BLOCK_CAUSAL, 0)
    with pytest.raises(TypeError):
        attention(qb.astype(np.float32), qb, qb, 0.5)


# ---------------------------------------------------------------- block-sparse

from oracle import MASK_BLOCK_SPARSE, SPARSE_BLOCK  # noqa: E402


def expand_block_mask(bm, Sq, Skv):
    """[B,H,nqb,nkb] block mask -> [B,H,Sq,Skv] boolean token mask."""
    t = torch.from_numpy(np.asarray(bm) != 0)
    t = t.repeat_interleave(SPARSE_BLOCK, dim=2).repeat_interleave(SPARSE_BLOCK, dim=3)
    return t[:, :, :Sq, :Skv]


def test_block_sparse_all_ones_is_full():
    rng = np.random.default_rng(40)
    B, H, Sq, Skv, D = 1, 2, 300, 270, 16
    qb, kb, vb = rand_bits(rng, (B, Sq, H, D)), rand_bits(rng, (B, Skv, H, D)), rand_bits(rng, (B, Skv, H, D))
    ones = np.ones((B, H, 3, 3), np.uint8)
    o, lse = attention(qb, kb, vb, 0.25, MASK_BLOCK_SPARSE, block_mask=ones)
    o_f, l_f = attention(qb, kb, vb, 0.25, MASK_CROSS)
    np.testing.assert_array_equal(o, o_f)
    np.testing.assert_array_equal(lse, l_f)


def test_block_sparse_block_causal_pattern_is_block_causal():
    rng = np.random.default_rng(41)
    B, H, S, D, c = 1, 2, 600, 16, 256  # chunks of two 128-token blocks
    qb, kb, vb = (rand_bits(rng, (B, S, H, D)) for _ in range(3))
    nb = -(-S // SPARSE_BLOCK)
    qi = np.arange(nb)[:, None] * SPARSE_BLOCK // c
    kj = np.arange(nb)[None, :] * SPARSE_BLOCK // c
    bm = np.broadcast_to((kj <= qi).astype(np.uint8), (B, H, nb, nb))
    o, lse = attention(qb, kb, vb, 0.3, MASK_BLOCK_SPARSE, block_mask=bm)
    o_c, l_c = attention(qb, kb, vb, 0.3, MASK_BLOCK_CAUSAL, c)
    np.testing.assert_array_equal(o, o_c)
    np.testing.assert_array_equal(lse, l_c)


def test_block_sparse_matches_torch_sdpa_with_the_expanded_mask():
    rng = np.random.default_rng(42)
    B, H, Sq, Skv, D = 2, 2, 400, 333, 16
    qb, kb, vb = rand_bits(rng, (B, Sq, H, D)), rand_bits(rng, (B, Skv, H, D)), rand_bits(rng, (B, Skv, H, D))
    bm = (rng.random((B, H, 4, 3)) < 0.5).astype(np.uint8)
    bm[0, 0, 1, :] = 0  # one query block of one head attends to nothing
    bm[1, 1, :, 2] = 1
    o, lse = attention(qb, kb, vb, 0.25, MASK_BLOCK_SPARSE, block_mask=bm)
    mask = expand_block_mask(bm, Sq, Skv)
    has_key = mask.any(dim=-1).numpy()  # [B,H,Sq]
    o_ref, l_ref = sdpa_reference(qb, kb, vb, 0.25, mask)
    for b in range(B):
        for h in range(H):
            rows = has_key[b, h]
            np.testing.assert_allclose(o[b, rows, h], o_ref[b, rows, h], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h, rows], l_ref[b, h, rows], rtol=0, atol=1e-12)
            assert np.all(o[b, ~rows, h] == 0.0) and np.all(np.isneginf(lse[b, h, ~rows]))
    assert (~has_key).any()


def test_block_sparse_rejects_a_wrong_mask_shape():
    qb = np.zeros((1, 200, 1, 8), np.uint16)
    with pytest.raises(ValueError):
        attention(qb, qb, qb, 0.5, MASK_BLOCK_SPARSE, block_mask=np.ones((1, 1, 1, 1)))


# ---------------------------------------------------------------------------
# Per-head Q/K RMS norm (the fused prologue's reference) and bf16 rounding.
# ---------------------------------------------------------------------------
from oracle import rms_norm, round_to_bf16_bits  # noqa: E402


def test_bf16_rounding_matches_torch_cast_and_ties_go_to_even():
    g = torch.Generator().manual_seed(31)
    x = torch.randn(4096, generator=g, dtype=torch.float32) * 7.0
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(round_to_bf16_bits(x.double().numpy()), want)
    ulp = 2.0 ** -7                               # bf16 spacing in [1, 2)
    ties = np.array([1 + ulp / 2, 1 + 3 * ulp / 2, -(1 + ulp / 2), 2 + 2 * ulp])  # the last is exact
    got = bits_to_float(round_to_bf16_bits(ties))
    assert got.tolist() == [1.0, 1 + 2 * ulp, -1.0, 2 + 2 * ulp]


def test_rms_norm_of_a_constant_row_and_a_one_hot_row():
    D = 128
    x = np.zeros((1, 2, 1, D), np.float64)
    x[0, 0, 0, :] = -3.0
    x[0, 1, 0, 5] = 2.0
    eps = 1e-6
    y = rms_norm(to_bf16_bits(x), eps=eps)
    assert np.allclose(y[0, 0, 0], -3.0 / math.sqrt(9.0 + eps), rtol=1e-15)
    expect = np.zeros(D)
    expect[5] = 2.0 / math.sqrt(4.0 / D + eps)      # = sqrt(D) as eps -> 0
    assert np.allclose(y[0, 1, 0], expect, rtol=1e-15, atol=0)


def test_rms_norm_output_has_unit_rms_and_ignores_power_of_two_scale():
    g = torch.Generator().manual_seed(32)
    x = (torch.randn(2, 9, 3, 128, generator=g, dtype=torch.float64) * 4).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    y = rms_norm(xb, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-13)
    x8 = (x.double() * 8).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)  # exact in bf16
    assert np.allclose(rms_norm(x8, eps=0.0), y, rtol=1e-13)


def test_rms_norm_per_head_weight_matches_torch_rms_norm_head_by_head():
    g = torch.Generator().manual_seed(33)
    x = torch.randn(1, 17, 4, 128, generator=g, dtype=torch.float64).to(torch.bfloat16)
    w = torch.rand(4, 128, generator=g, dtype=torch.float64) + 0.5
    y = rms_norm(x.view(torch.int16).numpy().view(np.uint16), w.numpy(), eps=1e-6)
    for h in range(4):
        ref = torch.nn.functional.rms_norm(x[:, :, h].double(), (128,), weight=w[h], eps=1e-6)
        assert np.allclose(y[:, :, h], ref.numpy(), rtol=1e-13, atol=1e-15)
    with pytest.raises(ValueError):
        rms_norm(x.view(torch.int16).numpy().view(np.uint16), w[:3].numpy())
