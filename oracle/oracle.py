"""ctypes front end of the fp64 C oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: see the package docstring.  Builds ``liboracle.so``
next to this file with gcc (OpenMP) on first use, then calls
``vdit_oracle_attn``.  Inputs are numpy ``uint16`` arrays holding bf16 bit
patterns in ``[B, S, H, D]`` layout; outputs are float64.

The arithmetic follows the plain definition of attention (see the C file's
header): softmax(scale * Q K^T) V over the allowed keys of each row, with the
natural-log LSE.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

MASK_FULL = 0
MASK_BLOCK_CAUSAL = 1
MASK_CROSS = 2
MASK_BLOCK_SPARSE = 3
SPARSE_BLOCK = 128

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_handle = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (gcc -O2 -fopenmp); returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        # -ffp-contract=off: no fused multiply-add, so each product is rounded
        # as written; -fno-fast-math keeps IEEE semantics for exp/log.
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _lib():
    global _handle
    with _lock:
        if _handle is None:
            build()
            h = ctypes.CDLL(_LIB)
            h.vdit_oracle_attn.restype = ctypes.c_int
            h.vdit_oracle_attn.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_int64,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ]
            h.vdit_oracle_max_threads.restype = ctypes.c_int
            _handle = h
    return _handle


def max_threads() -> int:
    """Threads the oracle's OpenMP runtime uses by default."""
    return int(_lib().vdit_oracle_max_threads())


def _as_bits(x) -> np.ndarray:
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (numpy uint16)")
    if a.ndim != 4:
        raise ValueError("oracle inputs are [B, S, H, D]")
    return a


def attention(q_bits, k_bits, v_bits, scale: float, mask_kind: int = MASK_FULL,
              chunk_tokens: int = 0, rows=None, threads: int = 0, block_mask=None):
    """fp64 attention.

    q_bits: [B, Sq, H, D] uint16 (bf16 bits); k_bits, v_bits: [B, Skv, H, D].
    rows: None for every row, else an int array of shape [n, 3] of (b, h, i).
    block_mask: for MASK_BLOCK_SPARSE, [B, H, ceil(Sq/128), ceil(Skv/128)]
    (nonzero = the query block attends to the key block).
    Returns (O, LSE): O is [B, Sq, H, D] float64 (all rows) or [n, D];
    LSE is [B, H, Sq] float64 (all rows) or [n].
    """
    q = _as_bits(q_bits)
    k = _as_bits(k_bits)
    v = _as_bits(v_bits)
    B, Sq, H, D = q.shape
    if k.shape[0] != B or k.shape[2] != H or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("K/V shapes do not match Q")
    Skv = k.shape[1]
    if rows is None:
        sel = None
        n = B * H * Sq
    else:
        sel = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = sel.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    mask = None
    if mask_kind == MASK_BLOCK_SPARSE:
        nqb, nkb = -(-Sq // SPARSE_BLOCK), -(-Skv // SPARSE_BLOCK)
        mask = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
        if mask.shape != (B, H, nqb, nkb):
            raise ValueError(f"block_mask must be [B, H, {nqb}, {nkb}]")
    rc = _lib().vdit_oracle_attn(
        q.ctypes.data, k.ctypes.data, v.ctypes.data,
        B, H, Sq, Skv, D, float(scale), int(mask_kind), int(chunk_tokens),
        None if mask is None else mask.ctypes.data,
        None if sel is None else sel.ctypes.data, n,
        o.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if rows is None:
        # rows were produced in (b, h, i) order
        o = o.reshape(B, H, Sq, D).transpose(0, 2, 1, 3).copy()
        lse = lse.reshape(B, H, Sq)
    return o, lse


def round_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even); returns the bit patterns.

    bf16 keeps 8 significant bits: with x = m * 2^e, 0.5 <= |m| < 1, the
    rounded value is rint(m * 2^8) * 2^(e - 8), where rint rounds half to even.
    Finite, normal-range inputs only (the RMS-normalised tensors this serves).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # exactly representable in binary32
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def rms_norm(x_bits, weight=None, eps: float = 1e-6) -> np.ndarray:
    """Per-(token, head) RMS norm of a bf16 [B, S, H, D] tensor, in float64.

    y[b, s, h, :] = x / sqrt(mean_d(x^2) + eps) * weight[h, :]  (weight None = 1).

    The pages name normalisation only as one of the parts of a DiT forward
    pass whose cost grows linearly with the latent patch count (gonka
    discussion #1155 on DiT support, "Pricing policy").  Read here as the
    per-head query/key RMS norm of the Wan2.x blocks that page proposes to
    serve: one learned weight per (head, channel), applied right before
    attention.  The attention then takes the result rounded to bf16
    (round_to_bf16_bits), the operand type of its bf16 products.
    """
    a = _as_bits(x_bits)
    x = (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if weight is not None:
        w = np.asarray(weight, dtype=np.float64)
        if w.shape != a.shape[2:]:
            raise ValueError("weight is [H, D]")
        y = y * w
    return y
