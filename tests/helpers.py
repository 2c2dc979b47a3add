"""Test helpers: bf16 conversion and the parity checker.

The checker holds the graded bars: max|err| <= 1e-2 (or one bf16 ulp of the
reference where |O| >= 2) and mean|err| <= 1e-3 on bf16 O against the fp64
oracle rounded to bf16, relative error <= 1e-3 on the
fp32 LSE (relative to max(|LSE|, 1)).  Because attention outputs shrink like sqrt(e / Skv) at long
sequences, it adds two scale-aware bars that an all-zero or shuffled O cannot
pass: rms(err) / rms(O_ref) <= 1e-2 per (b, h), and cosine(O, O_ref) >= 0.9999.
(bf16 rounding of O alone contributes about 2^-9 / sqrt(3) ~ 1e-3 to the first.)

It also measures max|err| / rms(O_ref) per (b, h), in three forms: against the
oracle rounded to bf16 (where a one-ulp rounding disagreement at the largest
|O| of a head counts in full), against the unrounded fp64 oracle (the
kernel's own error, its final bf16 rounding included), and the excess over
that rounding: max(|O - O_ref| - 2^-8 max(|O|, |O_ref|), 0) / rms(O_ref), since
rounding a value to bf16 moves it by at most 2^-8 of itself -- the last per
head, and per head dim against max(that dim's rms, the head's rms): a channel
whose values are several times larger than the rest (the value-outlier
channels of the 480p workload) has a proportionally larger error, and a
channel whose outputs barely vary over the rows (a tiny scale) has a tiny rms
of its own.  That last figure is held to EXCESS_BAR.  With the environment
variable VDIT_PARITY_REPORT set to a file path, every call appends its
measured figures to that file as one JSON line.
"""
import json
import os

import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_REL = 1e-3
REL_RMS_ERR = 1e-2
MIN_COSINE = 0.9999
# max(|O - O_ref| - 2^-8 max(|O|, |O_ref|), 0), the error beyond one bf16
# rounding of the output, over max(rms of the head dim, rms of the head) per
# (b, h): SURVEY's 2e-2 on max|err| / rms, read as a bar on what the output
# rounding does not explain.  For outputs that are one kernel's fp32 result
# rounded once to bf16; results composed of several rounded outputs (merged
# partials, other arithmetic) pass excess_bar=None.
EXCESS_BAR = 2e-2


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


def check_parity(o_gpu, o_ref, lse_gpu, lse_ref, group_rows=None, label="", excess_bar=EXCESS_BAR):
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
    err_exact = np.abs(o_gpu - np.asarray(o_ref, dtype=np.float64))
    excess = np.maximum(err_exact - 2.0 ** -8 * np.maximum(np.abs(o_gpu), np.abs(np.asarray(o_ref, np.float64))),
                        0.0)
    worst_rel = worst_max_rms = worst_max_rms_exact = worst_excess = worst_excess_ch = 0.0
    for g in groups:
        rms = max(float(np.sqrt(np.mean(o_ref[g] ** 2))), 1e-30)
        rms_err = float(np.sqrt(np.mean(err[g] ** 2)))
        worst_rel = max(worst_rel, rms_err / rms)
        worst_max_rms = max(worst_max_rms, float(err[g].max()) / rms)
        worst_max_rms_exact = max(worst_max_rms_exact, float(err_exact[g].max()) / rms)
        worst_excess = max(worst_excess, float(excess[g].max()) / rms)
        # per head dim, against max(its own rms over the group's rows, the head's rms)
        rms_ch = np.maximum(np.sqrt(np.mean(np.asarray(o_ref[g], np.float64) ** 2, axis=0)), rms)
        worst_excess_ch = max(worst_excess_ch, float((excess[g] / rms_ch).max()))
    res["rel_rms_err"] = worst_rel
    res["max_over_rms"] = worst_max_rms
    res["max_over_rms_exact"] = worst_max_rms_exact
    res["max_excess_over_rms"] = worst_excess
    res["max_excess_over_channel_rms"] = worst_excess_ch
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
          and (lse_gpu is None or res["lse_rel"] <= LSE_REL)
          and (excess_bar is None or worst_excess_ch <= excess_bar))
    res["ok"] = bool(ok)
    res["label"] = label
    report = os.environ.get("VDIT_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps(res) + "\n")
    return res


# ---------------------------------------------------------------- 8-bit path against the plain ExpCast statement
#
# The 8-bit kernel takes each probability byte against a reference of its own
# schedule (per 128-key tile, raised lazily, on a grid), the plain statement
# (oracle.fp8_oracle.attention_fp8_plain) against the row's true maximum.  For
# one key with exact probability 2^(u/8) (u in code units below the row max),
# ExpCast decodes to 2^(u/8) r(u), with ln r(u) = ln value(rint(u + 95.65)) -
# (u/8 + 5) ln 2 the byte map's own log error; a reference shifted by s gives
# r(u - s) instead.  So the two probabilities differ by a factor e^lambda with
# lambda = ln r(u - s) - ln r(u), whose spread is at most twice that of ln r:
# sigma_lambda <= 2 SIGMA_LN_R.  SIGMA_LN_R is the standard deviation of ln r
# over the normal codes (0.0312, pinned in tests/test_fp8_oracle_pins.py
# against the byte map, itself pinned to the page's 79.6% / one-code figures).
# To first order the outputs then differ by
#   O_k - O_p = sum_j w_j (lambda_j - mean lambda) (v_j - O_p),
# a sum of many small independent terms (lambda depends on the logits, v is
# drawn independently of them), with standard deviation at most
# sigma_lambda * spread, spread = sqrt(sum_j w_j^2 (v_j - O_p)^2) per row and
# head dim, computed by the plain oracle.  Likewise LSE_k - LSE_p = ln sum_j
# w_j e^lambda_j, within sigma_lambda sqrt(sum_j w_j^2) of the mean of lambda,
# which is zero over a uniform spread of u.  The bars:
#   per element  |O_k - O_p| <= 8 sigma_lambda spread + 2^-7 |O_p| + 1e-6
#                (8 standard deviations; 2^-7 |O|: the kernel's bf16 output,
#                one ulp, since its fp32 value may sit on the far side of a
#                rounding boundary from the plain value)
#   per (b, h)   rms(O_k - O_p) <= sigma_lambda rms(spread) + 2^-9 rms(O_p)
#   per row      |LSE_k - LSE_p| <= 8 sigma_lambda sqrt(sum_j w_j^2) + 1e-4
SIGMA_LN_R = 0.0313
SIGMA_LAMBDA = 2.0 * SIGMA_LN_R
EXPCAST_K = 8.0


def check_expcast_parity(o_gpu, o_plain, lse_gpu, lse_plain, spread_o, spread_l, group_rows=None, label=""):
    """Compare the 8-bit path's outputs with the plain ExpCast statement under the
    bars derived above.  o_*: [n, D]; lse_*, spread_l: [n]; spread_o: [n, D]."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_plain = np.asarray(o_plain, dtype=np.float64)
    d = np.abs(o_gpu - o_plain)
    bound = EXPCAST_K * SIGMA_LAMBDA * spread_o + 2.0 ** -7 * np.abs(o_plain) + 1e-6
    res = {"label": label, "max_over_bound": float((d / bound).max()),
           "max_d_over_spread": float((d / np.maximum(spread_o, 1e-30)).max())}
    groups = group_rows if group_rows is not None else [np.arange(o_gpu.shape[0])]
    worst = 0.0
    worst_rel = 0.0
    for g in groups:
        rms_d = float(np.sqrt(np.mean(d[g] ** 2)))
        bar = SIGMA_LAMBDA * float(np.sqrt(np.mean(spread_o[g] ** 2))) + 2.0 ** -9 * float(
            np.sqrt(np.mean(o_plain[g] ** 2)))
        worst = max(worst, rms_d / bar)
        worst_rel = max(worst_rel, rms_d / max(float(np.sqrt(np.mean(o_plain[g] ** 2))), 1e-30))
    res["rms_over_bar"] = worst
    res["rel_rms"] = worst_rel
    ok = res["max_over_bound"] <= 1.0 and worst <= 1.0
    if lse_gpu is not None:
        dl = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_plain, dtype=np.float64))
        lbound = EXPCAST_K * SIGMA_LAMBDA * np.asarray(spread_l) + 1e-4
        res["lse_over_bound"] = float((dl / lbound).max())
        res["lse_max_abs"] = float(dl.max())
        ok = ok and res["lse_over_bound"] <= 1.0
    res["ok"] = bool(ok)
    report = os.environ.get("VDIT_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps(res) + "\n")
    return res
