"""Algorithmic work counts for the roofline: FLOPs and compulsory HBM bytes.

Counts follow the plain definition of attention: for every allowed
(query, key) pair, D multiply-adds for the logit and D for the weighted value
sum, i.e. 4*D FLOPs a pair.  With S = 75,600 tokens and d = H*D = 5120 this is
4*S^2*d = 117.05 TFLOP, the score-matrix share of the ~133 TFLOP self-attention
figure in "Realtime video generation: FLOPS calculation and optimizations"
(sudonull.com), FLOP list (the rest is the Q/K/V/O projections, 8*S*d^2).
"""
from __future__ import annotations

from .workloads import MASK_BLOCK_CAUSAL, MASK_BLOCK_SPARSE, SPARSE_BLOCK, Attn


def allowed_pairs(Sq: int, Skv: int, mask_kind: int, chunk_tokens: int = 0) -> int:
    """Number of (query, key) pairs the mask allows, for the FLOP count."""
    if mask_kind == MASK_BLOCK_CAUSAL:
        c = int(chunk_tokens)
        total = 0
        for start in range(0, Sq, c):
            rows = min(c, Sq - start)
            total += rows * min(Skv, start + c)
        return total
    return Sq * Skv


def sparse_allowed_pairs(block_mask, Sq: int, Skv: int) -> int:
    """Allowed (query, key) pairs of a [B, H, nqb, nkb] block mask, summed over B and H."""
    import numpy as np
    m = np.asarray(block_mask) != 0
    nqb, nkb = m.shape[-2], m.shape[-1]
    rows = np.minimum(SPARSE_BLOCK, Sq - SPARSE_BLOCK * np.arange(nqb))  # tokens per query block
    cols = np.minimum(SPARSE_BLOCK, Skv - SPARSE_BLOCK * np.arange(nkb))
    return int(np.einsum("bhqk,q,k->", m.astype(np.int64), rows, cols))


def attn_flops(call: Attn, block_mask=None) -> float:
    """Algorithmic FLOPs of one call: 2*D for QK^T plus 2*D for PV per pair."""
    if call.mask_kind == MASK_BLOCK_SPARSE:
        return 4.0 * call.D * sparse_allowed_pairs(block_mask, call.Sq, call.Skv)
    return 4.0 * call.B * call.H * call.D * allowed_pairs(
        call.Sq, call.Skv, call.mask_kind, call.chunk_tokens)


def attn_min_bytes(call: Attn, with_lse: bool = True) -> float:
    """Compulsory HBM bytes of one call: Q, K, V read once, O (and LSE) written."""
    e = 2  # bf16
    b = call.B * call.H * call.D * e * (2 * call.Sq + 2 * call.Skv)
    if with_lse:
        b += call.B * call.H * call.Sq * 4
    return float(b)
