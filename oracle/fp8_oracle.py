"""Oracle of the 8-bit attention path: E4M3 quantisation, V-Smooth, ExpCast-FP8.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain numpy, written
from "VC-Attention: revolution in video generation speed without retraining"
(aikraft.ru), sections 02 "V-Smooth" and 03 "ExpCast-FP8":

* Q and K are quantised to E4M3 per 128-token block of one (batch, head)
  with an absmax scale (the page calls the kernel "8-bit" and E4M3 its code;
  the block is the "hardware block of 128 tokens" of section 02).
* V-Smooth: per 128-token block the mean is subtracted ("Demean") and only
  the residual is quantised, per channel, to E4M3; the mean is added back
  through the softmax row sum ("Restore").  The "Group" step (k-means
  permutation of K and V together) leaves non-causal attention unchanged and
  is not part of this function.
* ExpCast-FP8: the E4M3 byte of p = 2^x is written directly from the
  log-domain score as rint(8 * log2(v) + 56 + beta), beta = -0.35, instead of
  computing exp in fp32 and casting.

Readings where the page is silent (each one is listed with the design notes):
the probabilities are scaled by 2^P_SHIFT before coding so that the typical
values use E4M3's normal range; the running reference max is kept in code
units (8 x log2) on the grid N + frac(C) so that the FMA's addend is an
integer; the reference is raised when a tile's max exceeds it by more than
RESCALE_CODES; the per-channel V scale is shared by all blocks of a head and
floored at 2^-8 of the largest block mean.

Two statements of the attention are given.  ``attention_fp8_plain`` is the
page's ExpCast as stated: every byte against its row's true maximum, no
tiles, no running reference -- the independent check of the kernel's
attention.  ``attention_fp8`` walks the keys in 128-key tiles with a lazily
raised reference on a grid, the schedule the kernel uses, so that the
kernel's probability bytes can be checked one for one as a second, tighter
test; it is not an independent statement of the method.

Where floating point decides a stored code (the quantised Q, K, V and the
scales), this module uses the same fp32 operations as the kernel, so those
codes must match bit for bit.  The attention itself is computed in float64
from those codes; its probability codes can differ from the kernel's by one
in rare ties (the kernel's logits come out of an fp32 accumulator), which is
why attention outputs are compared with a tolerance.
"""
from __future__ import annotations

import math

import numpy as np

from .oracle import MASK_BLOCK_CAUSAL, MASK_CROSS, MASK_FULL, round_to_bf16_bits

E4M3_MAX = 448.0
BLOCK = 128
EXPCAST_BIAS = 56.0      # an E4M3 byte read as an integer is about 8 log2(v) + 56
EXPCAST_BETA = -0.35     # centres the remaining error
P_SHIFT = 5              # probabilities are coded as p * 2^P_SHIFT
RESCALE_CODES = 24.0     # 3 in log2 units: largest code 8*(3+5)+56-0.35 -> 120 <= 126
CODE_OFFSET = 8.0 * P_SHIFT + EXPCAST_BIAS + EXPCAST_BETA   # 95.65
_OFFSET_FRAC = CODE_OFFSET - math.floor(CODE_OFFSET)          # 0.65
MU_FLOOR = 2.0 ** -8     # V channel scale >= 2^-8 x largest |block mean| / 448
LOG2E = 1.4426950408889634


# ------------------------------------------------------------------ E4M3

def e4m3_codes(x) -> np.ndarray:
    """float32 values -> E4M3 (fn variant) byte codes, round to nearest even,
    finite values beyond +-448 saturate to +-448.

    E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; normals
    (1 + m/8) 2^(e-7) for e = 1..15 (0x7F is NaN, so 448 = 1.75 * 2^8 is the
    largest), subnormals m/8 * 2^-6.  The quantum of a normal value in
    [2^E, 2^(E+1)) is 2^(E-3); every subnormal has quantum 2^-9.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_codes takes finite values")
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, e = np.frexp(a)                      # a = m 2^e, 0.5 <= m < 1
    quantum_exp = np.where(a >= 2.0 ** -6, e - 1 - 3, -9)
    r = np.ldexp(np.rint(np.ldexp(a, -quantum_exp)), quantum_exp)   # exact in float64
    r = np.minimum(r, E4M3_MAX)
    _, er = np.frexp(r)
    E = er - 1
    normal = r >= 2.0 ** -6
    mant = np.where(normal, np.ldexp(r, -E) - 1.0, 0.0) * 8.0
    code = np.where(normal, ((E + 7) << 3) + mant.astype(np.int64), np.ldexp(r, 9).astype(np.int64))
    code = np.where(r == 0, 0, code)
    return (code.astype(np.int64) | (np.signbit(x).astype(np.int64) << 7)).astype(np.uint8)


def e4m3_values(codes) -> np.ndarray:
    """E4M3 byte codes -> their exact values (float64)."""
    c = np.asarray(codes, dtype=np.int64)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, np.ldexp(m.astype(np.float64), -9), np.ldexp(1.0 + m / 8.0, e - 7))
    if np.any((c & 0x7F) == 0x7F):
        raise ValueError("NaN code")
    return np.where(c & 0x80, -mag, mag)


def _bf16_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _padded_blocks(x32: np.ndarray) -> np.ndarray:
    """[B, S, H, D] -> [B, H, nb, 128, D] with zero rows past S."""
    B, S, H, D = x32.shape
    nb = -(-S // BLOCK)
    pad = np.zeros((B, nb * BLOCK, H, D), dtype=np.float32)
    pad[:, :S] = x32
    return pad.reshape(B, nb, BLOCK, H, D).transpose(0, 3, 1, 2, 4)


# ------------------------------------------------------------------ Q and K

def quantize_qk(x_bits):
    """Per-block E4M3 quantisation of Q or K (bf16 bits, [B, S, H, D]).

    For each (b, h, block of 128 tokens): amax = max |x| (fp32),
    scale = amax / 448, and code = E4M3(x * (448 / amax)) with both
    quotients and the product rounded to fp32 (zero block: scale 0, codes 0).
    Returns (codes uint8 [B, S, H, D], scale float32 [B, H, nb]).
    """
    x = _bf16_to_f32(x_bits)
    B, S, H, D = x.shape
    xb = _padded_blocks(x)                                    # [B, H, nb, 128, D]
    amax = np.abs(xb).max(axis=(3, 4)).astype(np.float32)    # [B, H, nb]
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0)).astype(np.float32)
    y = (xb * inv[:, :, :, None, None]).astype(np.float32)
    codes = e4m3_codes(y).reshape(B, H, -1, D)[:, :, :S]      # [B, H, S, D]
    return np.ascontiguousarray(codes.transpose(0, 2, 1, 3)), scale


# ------------------------------------------------------------------ V-Smooth

def vsmooth(v_bits):
    """V-Smooth Demean + per-channel E4M3 quantisation of V (bf16 bits, [B, S, H, D]).

    mu[b,h,blk,d]  = (sequential fp32 sum of the block's valid tokens) / n
    R              = v - mu                                           (fp32)
    amax[b,h,d]    = max(max_tokens |R|, 2^-8 * max_blocks |mu|)
    scale[b,h,d]   = amax / 448;  code = E4M3(R * (448 / amax))      (fp32 steps)
    mu'            = mu * (448 / amax), split as bf16 hi + bf16 lo (the kernel's
                     restore operand; mu' * scale ~ mu)
    Returns a dict with codes [B, S, H, D] (uint8), scale [B, H, D] (f32),
    mu [B, H, nb, D] (f32), mu_hi / mu_lo [B, H, nb, D] (bf16 bits).
    """
    v = _bf16_to_f32(v_bits)
    B, S, H, D = v.shape
    vb = _padded_blocks(v)                                    # [B, H, nb, 128, D]
    nb = vb.shape[2]
    n = np.full(nb, BLOCK, dtype=np.int64)
    n[-1] = S - (nb - 1) * BLOCK
    sums = np.cumsum(vb, axis=3, dtype=np.float32)            # sequential fp32 running sums
    total = np.stack([sums[:, :, i, n[i] - 1] for i in range(nb)], axis=2)    # [B, H, nb, D]
    mu = (total / n.astype(np.float32)[None, None, :, None]).astype(np.float32)
    valid = (np.arange(BLOCK)[None, :] < n[:, None])          # [nb, 128]
    R = np.where(valid[None, None, :, :, None], (vb - mu[:, :, :, None, :]).astype(np.float32), np.float32(0))
    amax_r = np.abs(R).max(axis=(2, 3)).astype(np.float32)    # [B, H, D]
    amax_mu = np.abs(mu).max(axis=2).astype(np.float32)
    amax = np.maximum(amax_r, (amax_mu * np.float32(MU_FLOOR)).astype(np.float32))
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0)).astype(np.float32)
    y = (R * inv[:, :, None, None, :]).astype(np.float32)
    codes = e4m3_codes(y).reshape(B, H, nb * BLOCK, D)[:, :, :S].transpose(0, 2, 1, 3)
    mu_p = (mu * inv[:, :, None, :]).astype(np.float32)
    hi = round_to_bf16_bits(mu_p.astype(np.float64))
    lo = round_to_bf16_bits((mu_p - _bf16_to_f32(hi)).astype(np.float32).astype(np.float64))
    return {"codes": np.ascontiguousarray(codes), "scale": scale, "mu": mu, "mu_hi": hi, "mu_lo": lo}


# ------------------------------------------------------------------ ExpCast

def expcast_codes(z_minus_ref) -> np.ndarray:
    """ExpCast-FP8 bytes from (logit - reference) in code units (8 x log2).

    byte = rint(8 log2(p 2^P_SHIFT) + 56 + beta) = rint(z - ref + CODE_OFFSET),
    clamped below at 0 (-inf gives 0).  rint rounds half to even.
    """
    t = np.asarray(z_minus_ref, dtype=np.float64) + CODE_OFFSET
    y = np.rint(np.where(np.isneginf(t), 0.0, t))
    y = np.maximum(y, 0.0)
    if np.any(y > 126):
        raise ValueError("code above the E4M3 range: the reference max was not maintained")
    return y.astype(np.uint8)


def reference_for(zmax: float) -> float:
    """Smallest reference on the grid N + frac(CODE_OFFSET) that is >= zmax."""
    return math.ceil(zmax - _OFFSET_FRAC) + _OFFSET_FRAC


def expcast_row(z) -> np.ndarray:
    """ExpCast-FP8 bytes of one row of logits z (code units, 8 x log2; -inf
    where masked), taken against the row's own maximum, with no tiling:
    byte_j = rint(z_j - max z + CODE_OFFSET), clamped below at 0.  The largest
    logit gets rint(95.65) = 96, the byte of 2^P_SHIFT."""
    z = np.asarray(z, dtype=np.float64)
    return expcast_codes(z - z.max())


def _allowed_prefix(mask_kind, i, Skv, chunk):
    if mask_kind == MASK_BLOCK_CAUSAL:
        return min(Skv, (i // chunk + 1) * chunk)
    return Skv


def attention_fp8(q_bits, k_bits, v_bits, scale: float, mask_kind: int = MASK_FULL, chunk_tokens: int = 0,
                  rows=None, quantized=None):
    """The 8-bit attention (E4M3 Q/K/V with V-Smooth, ExpCast-FP8 probabilities), float64.

    Per query row i of (b, h), key tiles j of 128 are visited in order:
      z      = 8 log2(e) scale sq sk (q_codes . k_codes)     (code units; -inf where masked)
      ref    = reference_for(max z) on the first tile; later raised to
               reference_for(max z) only when max z > ref + RESCALE_CODES, with
               the running sums multiplied by 2^((ref_old - ref_new)/8)
      c      = expcast_codes(z - ref);   p_j = value(c_j)
      l     += sum_j p_j
      acc   += sum_j p_j * (code_v[j] * scale_v) + (sum_j p_j) * mu_block
    O = acc / l,  LSE = ln 2 * (ref/8 - P_SHIFT + log2 l).
    Returns (O, LSE) shaped like oracle.attention: [B, Sq, H, D] and [B, H, Sq],
    or [n, D] and [n] for the (b, h, i) triples in `rows`.
    """
    if quantized is None:
        quantized = (quantize_qk(q_bits), quantize_qk(k_bits), vsmooth(v_bits))
    (qc, qs), (kc, ks), vs = quantized
    B, Sq, H, D = qc.shape
    Skv = kc.shape[1]
    if mask_kind not in (MASK_FULL, MASK_BLOCK_CAUSAL, MASK_CROSS):
        raise ValueError("mask kind")
    if mask_kind == MASK_BLOCK_CAUSAL and chunk_tokens < 1:
        raise ValueError("chunk_tokens")
    qv = e4m3_values(qc)
    kv = e4m3_values(kc)
    vdeq = e4m3_values(vs["codes"]) * vs["scale"].astype(np.float64)[:, None, :, :]   # [B, Skv, H, D]
    mu = vs["mu"].astype(np.float64)                                                  # [B, H, nb, D]
    if rows is None:
        sel = [(b, h, i) for b in range(B) for h in range(H) for i in range(Sq)]
    else:
        sel = [tuple(int(t) for t in r) for r in np.asarray(rows).reshape(-1, 3)]
    o = np.zeros((len(sel), D))
    lse = np.zeros(len(sel))
    c0 = 8.0 * LOG2E * float(scale)
    for r, (b, h, i) in enumerate(sel):
        n = _allowed_prefix(mask_kind, i, Skv, chunk_tokens)
        ref = None
        acc = np.zeros(D)
        ell = 0.0
        for j in range(-(-n // BLOCK)):
            k0, k1 = j * BLOCK, min((j + 1) * BLOCK, n)
            a = c0 * float(qs[b, h, i // BLOCK]) * float(ks[b, h, j])
            z = a * (kv[b, k0:k1, h, :] @ qv[b, i, h, :])
            zmax = float(z.max())
            if ref is None:
                ref = reference_for(zmax)
            elif zmax > ref + RESCALE_CODES:
                new = reference_for(zmax)
                f = 2.0 ** ((ref - new) / 8.0)
                acc *= f
                ell *= f
                ref = new
            p = e4m3_values(expcast_codes(z - ref))
            lb = float(p.sum())
            acc += p @ vdeq[b, k0:k1, h, :] + lb * mu[b, h, j]
            ell += lb
        o[r] = acc / ell
        lse[r] = math.log(2.0) * (ref / 8.0 - P_SHIFT + math.log2(ell))
    if rows is not None:
        return o, lse
    o_full = np.zeros((B, Sq, H, D))
    lse_full = np.zeros((B, H, Sq))
    for r, (b, h, i) in enumerate(sel):
        o_full[b, i, h] = o[r]
        lse_full[b, h, i] = lse[r]
    return o_full, lse_full


def attention_fp8_plain(q_bits, k_bits, v_bits, scale: float, mask_kind: int = MASK_FULL, chunk_tokens: int = 0,
                        rows=None, quantized=None, spread: bool = False):
    """The 8-bit attention with ExpCast-FP8 as the VC-Attention page states it:
    every probability byte is taken against its row's true maximum.

    This is the plain statement of section 03 ("ExpCast-FP8") on the operands
    of section 02 ("V-Smooth"), without any of a kernel's scheduling choices:
    no 128-key tiles, no lazily raised running reference, no reference grid.
    For each query row i of (b, h), over all of its allowed keys j at once:
      z_j    = 8 log2(e) scale sq sk_j (q_codes . k_codes_j)   (code units)
      byte_j = expcast_row(z)_j = rint(z_j - max z + 95.65), clamped at 0
      p_j    = value(byte_j) / 2^P_SHIFT       (2^P_SHIFT: reading of the page's range)
      v^_j   = value(code_v_j) scale_v + mu_block(j)   (V-Smooth's Demean undone: Restore)
    O = sum_j p_j v^_j / sum_j p_j,  LSE = ln 2 (max z / 8 + log2 sum_j p_j).
    The only readings it shares with attention_fp8 are those of the operands
    (E4M3 blocks, V-Smooth's scales) and of the byte map (P_SHIFT, beta).

    spread=True also returns, per row and head dim, sqrt(sum_j w_j^2 (v^_jd - O_d)^2)
    with w_j = p_j / sum p -- the size of the O perturbation that independent
    relative errors of one unit in the probabilities would cause -- and per
    row sqrt(sum_j w_j^2), its counterpart for LSE.
    Returns (O, LSE[, spread_o, spread_lse]) shaped like attention_fp8.
    """
    if quantized is None:
        quantized = (quantize_qk(q_bits), quantize_qk(k_bits), vsmooth(v_bits))
    (qc, qs), (kc, ks), vs = quantized
    B, Sq, H, D = qc.shape
    Skv = kc.shape[1]
    if mask_kind not in (MASK_FULL, MASK_BLOCK_CAUSAL, MASK_CROSS):
        raise ValueError("mask kind")
    if mask_kind == MASK_BLOCK_CAUSAL and chunk_tokens < 1:
        raise ValueError("chunk_tokens")
    qv = e4m3_values(qc)
    kv = e4m3_values(kc)
    blk = np.arange(Skv) // BLOCK
    v_hat = (e4m3_values(vs["codes"]) * vs["scale"].astype(np.float64)[:, None, :, :]
             + vs["mu"].astype(np.float64)[:, :, blk, :].transpose(0, 2, 1, 3))          # [B, Skv, H, D]
    if rows is None:
        sel = [(b, h, i) for b in range(B) for h in range(H) for i in range(Sq)]
    else:
        sel = [tuple(int(t) for t in r) for r in np.asarray(rows).reshape(-1, 3)]
    o = np.zeros((len(sel), D))
    lse = np.zeros(len(sel))
    spr = np.zeros((len(sel), D)) if spread else None
    spl = np.zeros(len(sel)) if spread else None
    c0 = 8.0 * LOG2E * float(scale)
    for r, (b, h, i) in enumerate(sel):
        n = _allowed_prefix(mask_kind, i, Skv, chunk_tokens)
        a = c0 * float(qs[b, h, i // BLOCK]) * ks[b, h, blk[:n]].astype(np.float64)
        z = a * (kv[b, :n, h, :] @ qv[b, i, h, :])
        p = e4m3_values(expcast_row(z)) * 2.0 ** -P_SHIFT
        ell = float(p.sum())
        o[r] = p @ v_hat[b, :n, h, :] / ell
        lse[r] = math.log(2.0) * (float(z.max()) / 8.0 + math.log2(ell))
        if spread:
            w = p / ell
            spr[r] = np.sqrt((w[:, None] ** 2 * (v_hat[b, :n, h, :] - o[r]) ** 2).sum(axis=0))
            spl[r] = math.sqrt(float((w ** 2).sum()))
    if rows is not None:
        return (o, lse, spr, spl) if spread else (o, lse)
    o_full = np.zeros((B, Sq, H, D))
    lse_full = np.zeros((B, H, Sq))
    spr_full = np.zeros((B, Sq, H, D)) if spread else None
    spl_full = np.zeros((B, H, Sq)) if spread else None
    for r, (b, h, i) in enumerate(sel):
        o_full[b, i, h] = o[r]
        lse_full[b, h, i] = lse[r]
        if spread:
            spr_full[b, i, h] = spr[r]
            spl_full[b, h, i] = spl[r]
    return (o_full, lse_full, spr_full, spl_full) if spread else (o_full, lse_full)
