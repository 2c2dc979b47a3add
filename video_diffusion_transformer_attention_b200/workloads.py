"""Seeded synthetic workloads for the video-DiT attention forward pass.

This module only draws inputs.  It holds none of the attention arithmetic, so
the fp64 oracle and the CUDA path can both be fed from it without sharing any
of the method's code.

Shapes come from the pages' Wan-style workloads:

* 720p Wan2.1-14B: 21 latent frames x 3600 spatial tokens = 75,600 tokens,
  40 heads of 128 (d = 5120) -- "Realtime video generation: FLOPS calculation
  and optimizations" (sudonull.com), opening paragraph and the FLOP list.
* Wan2.2 with 16x16 spatial compression: 18,900 tokens -- same page, section
  "Why the VAE is the main lever of the future".
* 480p Wan2.1-1.3B: 21 x 30 x 52 = 32,760 tokens, 12 heads of 128.
* Block-causal chunks of 3 latent frames (num-frames divisible by 3) -- Wave
  Forcing digest (airadar.tv), usage notes; 3 x 1560 = 4680 tokens a chunk.
* Value outliers concentrated in a few channels that differ between heads --
  "VC-Attention" (aikraft.ru), section 02 "V-Smooth".

Recipe (the pages give shapes and value statistics but no generator, so the
choices below are this module's): a CPU ``torch.Generator`` seeded with
``1000 + config index`` draws Q, K, V (in that order) as N(0, 1) float32 in
[B, S, H, D] layout.  Where a workload says so, Q and K are RMS-normalised over
each (token, head) D-vector in float32 (``x / sqrt(mean(x^2) + 1e-6)``, weight
1), and 3 of the 128 V channels of each head -- picked by a seeded permutation
per head (round(2% of 128) = 3; the gain 8 is exact in bf16) -- are multiplied
by 8.  Everything is then rounded to bf16, and those
bf16 values are the inputs.  Cross-attention text K/V come from a second
generator seeded ``2000 + config index``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

MASK_FULL = 0
MASK_BLOCK_CAUSAL = 1
MASK_CROSS = 2
MASK_BLOCK_SPARSE = 3
SPARSE_BLOCK = 128

RMS_EPS = 1e-6
OUTLIER_CHANNELS = 3  # round(0.02 * 128)
OUTLIER_GAIN = 8.0


@dataclass(frozen=True)
class Attn:
    """One attention call of a workload."""
    name: str
    B: int
    H: int
    Sq: int
    Skv: int
    D: int
    mask_kind: int
    chunk_tokens: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


@dataclass(frozen=True)
class Workload:
    """A workload: its seed index, value recipe and one or more calls."""
    name: str
    index: int
    recipe: str  # "iid", "rms_qk", "rms_qk_vout"
    calls: tuple = field(default_factory=tuple)
    text_tokens: int = 0


WORKLOADS = {
    "pr1_s1024": Workload(
        "pr1_s1024", 0, "iid",
        (Attn("self", 1, 2, 1024, 1024, 128, MASK_FULL),)),
    "wan21_1p3b_480p": Workload(
        "wan21_1p3b_480p", 1, "rms_qk_vout",
        (Attn("self", 1, 12, 32760, 32760, 128, MASK_FULL),)),
    "wan22_720p_16x16": Workload(
        "wan22_720p_16x16", 2, "rms_qk",
        (Attn("self", 1, 40, 18900, 18900, 128, MASK_FULL),)),
    "wan21_14b_720p": Workload(
        "wan21_14b_720p", 3, "rms_qk",
        (Attn("self", 1, 40, 75600, 75600, 128, MASK_FULL),
         Attn("cross", 1, 40, 75600, 512, 128, MASK_CROSS)),
        text_tokens=512),
    "block_causal_7x4680": Workload(
        "block_causal_7x4680", 4, "rms_qk",
        (Attn("self", 1, 12, 32760, 32760, 128, MASK_BLOCK_CAUSAL, 4680),)),
    # block-sparse self-attention on the 720p Wan2.1-14B shape: each query
    # block keeps its own key block plus a seeded 25% of the others (the
    # page's "x4" for block-sparse attention read as keeping a quarter)
    "wan21_14b_720p_sparse25": Workload(
        "wan21_14b_720p_sparse25", 5, "rms_qk",
        (Attn("self", 1, 40, 75600, 75600, 128, MASK_BLOCK_SPARSE),)),
}

SPARSE_DENSITY = 0.25


def _rms_normalise(x: torch.Tensor) -> torch.Tensor:
    x = x.float()
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + RMS_EPS)


def _scale_outlier_channels(v: torch.Tensor, gen: torch.Generator) -> torch.Tensor:
    """Multiply OUTLIER_CHANNELS channels of every head by OUTLIER_GAIN."""
    H, D = v.shape[2], v.shape[3]
    gain = torch.ones(H, D, dtype=torch.float32)
    for h in range(H):
        ch = torch.randperm(D, generator=gen)[:OUTLIER_CHANNELS]
        gain[h, ch] = OUTLIER_GAIN
    return v * gain  # broadcast over [B, S]


def draw_qkv(B: int, H: int, Sq: int, Skv: int, D: int, seed: int,
             recipe: str = "iid", raw_qk: bool = False):
    """Draw bf16 (Q, K, V) on the CPU in [B, S, H, D] layout.

    raw_qk: skip the RMS norm of Q and K that the recipe asks for (the fused
    Q/K-norm entry point applies it inside the kernel instead)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    q = torch.randn((B, Sq, H, D), generator=gen, dtype=torch.float32)
    k = torch.randn((B, Skv, H, D), generator=gen, dtype=torch.float32)
    v = torch.randn((B, Skv, H, D), generator=gen, dtype=torch.float32)
    if recipe in ("rms_qk", "rms_qk_vout") and not raw_qk:
        q = _rms_normalise(q)
        k = _rms_normalise(k)
    if recipe == "rms_qk_vout":
        v = _scale_outlier_channels(v, gen)
    elif recipe not in ("iid", "rms_qk"):
        raise ValueError(f"unknown recipe {recipe!r}")
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def draw_text_kv(B: int, H: int, Skv: int, D: int, seed: int):
    """Cross-attention text K/V: raw N(0, 1), bf16, [B, Skv, H, D]."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    k = torch.randn((B, Skv, H, D), generator=gen, dtype=torch.float32)
    v = torch.randn((B, Skv, H, D), generator=gen, dtype=torch.float32)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def workload_inputs(name: str, raw_qk: bool = False):
    """All inputs of a named workload, as a dict of CPU bf16 tensors.

    Keys: "q", "k", "v" (self-attention) and, for workloads with a text
    sequence, "k_text", "v_text".
    """
    w = WORKLOADS[name]
    self_call = w.calls[0]
    q, k, v = draw_qkv(self_call.B, self_call.H, self_call.Sq, self_call.Skv,
                       self_call.D, 1000 + w.index, w.recipe, raw_qk)
    out = {"q": q, "k": k, "v": v}
    if self_call.mask_kind == MASK_BLOCK_SPARSE:
        out["block_mask"] = draw_block_mask(self_call.B, self_call.H, self_call.Sq, self_call.Skv,
                                            SPARSE_DENSITY, 3000 + w.index)
    if w.text_tokens:
        kt, vt = draw_text_kv(self_call.B, self_call.H, w.text_tokens,
                              self_call.D, 2000 + w.index)
        out["k_text"] = kt
        out["v_text"] = vt
    return out


def draw_block_mask(B: int, H: int, Sq: int, Skv: int, density: float, seed: int,
                    keep_diagonal: bool = True) -> torch.Tensor:
    """Seeded block mask [B, H, ceil(Sq/128), ceil(Skv/128)] uint8 (CPU).

    Each block is kept with probability `density`; with keep_diagonal the
    block pair (i, i) is always kept (a query block sees its own tokens).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    nqb, nkb = -(-Sq // SPARSE_BLOCK), -(-Skv // SPARSE_BLOCK)
    m = (torch.rand((B, H, nqb, nkb), generator=gen) < density)
    if keep_diagonal:
        d = torch.arange(min(nqb, nkb))
        m[:, :, d, d] = True
    return m.to(torch.uint8)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a CPU bf16 tensor as numpy uint16 (no copy of values)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def sample_rows(B: int, H: int, Sq: int, per_head: int, seed: int,
                chunk_tokens: int = 0, tile: int = 128):
    """Deterministic (b, h, i) row sample for large-shape parity checks.

    Every (b, h) gets the first and last rows, the rows on both sides of every
    tile boundary within the first and last two tiles, the last full tile,
    rows on both sides of every chunk boundary, and seeded-random rows up to
    ``per_head`` rows in total.
    """
    rng = np.random.default_rng(int(seed))
    fixed = {0, Sq - 1}
    for t in (1, 2, (Sq // tile) - 1, Sq // tile):
        for r in (t * tile - 1, t * tile):
            if 0 <= r < Sq:
                fixed.add(r)
    if chunk_tokens:
        for c in range(chunk_tokens, Sq, chunk_tokens):
            fixed.update((c - 1, c))
    fixed = np.array(sorted(fixed), dtype=np.int64)
    others = np.setdiff1d(np.arange(Sq, dtype=np.int64), fixed)
    extra = min(max(0, per_head - len(fixed)), len(others))
    rows = []
    for b in range(B):
        for h in range(H):
            rand = rng.choice(others, size=extra, replace=False) if extra else []
            for i in np.union1d(fixed, rand):
                rows.append((b, h, int(i)))
    return np.asarray(rows, dtype=np.int64)
