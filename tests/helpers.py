"""Test helpers: bf16 conversion and the parity checker.

The checker holds the graded bars: max|err| <= 1e-2 (or one bf16 ulp of the
reference where |O| >= 2) and mean|err| <= 1e-3 on bf16 O against the fp64
oracle rounded to bf16, relative error <= 1e-3 on the
fp32 LSE (relative to max(|LSE|, 1)).  Because attention outputs shrink like sqrt(e / Skv) at long
sequences, it adds two scale-aware bars that an all-zero or shuffled O cannot
pass: rms(err) / rms(O_ref) <= 1e-2 per (b, h), and cosine(O, O_ref) >= 0.9999.
(bf16 rounding of O alone contributes about 2^-9 / sqrt(3) ~ 1e-3 to the first.)
"""
import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_REL = 1e-3
REL_RMS_ERR = 1e-2
MIN_COSINE = 0.9999


def to_bf16_bits(x) -> np.ndarray:
    """float array -> bf16 bit patterns (round to nearest even), numpy uint16."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_float(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 (through float32), as float64."""
    return bits_to_float(to_bf16_bits(np.asarray(x, dtype=np.float64)))


def check_parity(o_gpu, o_ref, lse_gpu, lse_ref, group_rows=None, label=""):
    """Compare one call's outputs; returns a dict of the measured errors.

    o_gpu: [n, D] float (bf16 values), o_ref: [n, D] float64 oracle values.
    lse_*: [n].  group_rows: optional list of index arrays, one per (b, h), for
    the per-head relative bar (default: all rows form one group).
    """
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref_b = round_bf16(o_ref)
    err = np.abs(o_gpu - o_ref_b)
    # 1e-2 absolute, or one bf16 ulp of the reference value where that is
    # larger (|O| >= 2 only; the Wan workloads keep |O| well below 1)
    bound = np.maximum(MAX_ABS, np.abs(o_ref_b) * 2.0 ** -7)
    res = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
           "max_over_bound": float((err / bound).max())}
    groups = group_rows if group_rows is not None else [np.arange(o_gpu.shape[0])]
    worst_rel = 0.0
    for g in groups:
        rms = float(np.sqrt(np.mean(o_ref[g] ** 2)))
        rms_err = float(np.sqrt(np.mean(err[g] ** 2)))
        worst_rel = max(worst_rel, rms_err / max(rms, 1e-30))
    res["rel_rms_err"] = worst_rel
    a, b = o_gpu.ravel(), np.asarray(o_ref, dtype=np.float64).ravel()
    res["cosine"] = float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        # relative to |LSE|, floored at 1 so that an LSE near 0 (a short key
        # sequence with small logits) is held to 1e-3 absolute instead
        res["lse_rel"] = float(np.max(np.abs(lg - lr) / np.maximum(np.abs(lr), 1.0)))
    ok = (res["max_over_bound"] <= 1.0 and res["mean_abs"] <= MEAN_ABS
          and res["rel_rms_err"] <= REL_RMS_ERR and res["cosine"] >= MIN_COSINE
          and (lse_gpu is None or res["lse_rel"] <= LSE_REL))
    res["ok"] = bool(ok)
    res["label"] = label
    return res
