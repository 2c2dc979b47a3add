"""Oracle of V-Smooth's "Group" step: online k-means over value tokens, and the
joint permutation of K and V that puts each cluster's tokens together.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain numpy, float64,
from "VC-Attention: revolution in video generation speed without retraining"
(aikraft.ru), section 02 "V-Smooth", Group: value tokens of each batch and
head are clustered with an online k-means, and keys and values are permuted
together, which leaves non-causal attention unchanged; the grouping then
makes each 128-token block's mean (the Demean step) capture more of the
block, and it is rerun only on the first quarter of the denoising steps, the
permutation being reused for four neighbouring steps.

Read here as Lloyd's algorithm warm-started from the caller's centroids
("online" across denoising steps): each iteration assigns every token to its
nearest centroid in Euclidean distance (ties to the lowest index) and moves
every centroid to the mean of its tokens (a centroid without tokens stays).
The permutation lists the tokens of cluster 0 in token order, then those of
cluster 1, and so on (a stable sort by cluster).
"""
from __future__ import annotations

import numpy as np


def _as_f64(v_bits):
    v = np.asarray(v_bits, dtype=np.uint16)
    return (v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assign(v, centroids) -> np.ndarray:
    """Nearest centroid of every token.  v: [n, D] float64, centroids: [C, D].

    Squared distances are taken in float64; ties go to the lowest index."""
    v = np.asarray(v, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    d2 = ((v[:, None, :] - c[None, :, :]) ** 2).sum(axis=2)
    return np.argmin(d2, axis=1)


def distances(v, centroids) -> np.ndarray:
    """[n, C] squared Euclidean distances in float64."""
    v = np.asarray(v, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    return ((v[:, None, :] - c[None, :, :]) ** 2).sum(axis=2)


def update(v, labels, centroids) -> np.ndarray:
    """Each centroid moved to the mean of its tokens; empty clusters stay put."""
    v = np.asarray(v, dtype=np.float64)
    c = np.array(centroids, dtype=np.float64, copy=True)
    for k in range(c.shape[0]):
        m = labels == k
        if m.any():
            c[k] = v[m].mean(axis=0)
    return c


def group_permutation(labels) -> np.ndarray:
    """Stable sort of the tokens by cluster: perm[i] = token at position i."""
    return np.argsort(np.asarray(labels), kind="stable")


def kmeans(v_bits, centroids, iters: int):
    """Lloyd iterations per (b, h) on bf16 V ([B, S, H, D] bits).

    centroids: [B, H, C, D] float.  Returns (labels [B, H, S] from the last
    assignment, centroids after the last update, perm [B, H, S]).  With
    iters = 0 only the assignment and permutation of the given centroids."""
    v = _as_f64(v_bits)
    B, S, H, D = v.shape
    c = np.array(centroids, dtype=np.float64, copy=True)
    labels = np.zeros((B, H, S), dtype=np.int64)
    perm = np.zeros((B, H, S), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            x = v[b, :, h, :]
            for _ in range(iters):
                lab = assign(x, c[b, h])
                c[b, h] = update(x, lab, c[b, h])
            lab = assign(x, c[b, h])
            labels[b, h] = lab
            perm[b, h] = group_permutation(lab)
    return labels, c, perm


def permute_tokens(x_bits, perm) -> np.ndarray:
    """x[b, perm[b, h, i], h, :] gathered to position i, per head ([B, S, H, D])."""
    x = np.asarray(x_bits)
    B, S, H, D = x.shape
    out = np.empty_like(x)
    for b in range(B):
        for h in range(H):
            out[b, :, h, :] = x[b, perm[b, h], h, :]
    return out


def block_energy_removed(v, block: int = 128) -> float:
    """Share of V's energy removed by subtracting each block's mean (one head, [S, D])."""
    v = np.asarray(v, dtype=np.float64)
    S = v.shape[0]
    total = float((v ** 2).sum())
    removed = 0.0
    for t0 in range(0, S, block):
        blk = v[t0:t0 + block]
        mu = blk.mean(axis=0)
        removed += float((blk ** 2).sum() - ((blk - mu) ** 2).sum())
    return removed / total
