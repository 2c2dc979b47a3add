"""Pins of the 8-bit attention oracle (oracle/fp8_oracle.py) to facts outside it.

E4M3 rounding is pinned to torch's float8_e4m3fn cast; ExpCast-FP8 to the
figures the VC-Attention page prints (tests/golden/vc_attention_expcast.txt);
quantisation and V-Smooth to their error bounds and closed forms; the whole
attention to closed forms and to the exact float64 attention of oracle.oracle.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import MASK_BLOCK_CAUSAL, MASK_FULL, attention
from oracle import fp8_oracle as f8
from tests.helpers import bits_to_float, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "vc_attention_expcast.txt")


def golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def torch_e4m3(x32):
    return torch.tensor(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# ------------------------------------------------------------------ E4M3

def test_e4m3_rounding_matches_torch_cast():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(20000) * 40, g.standard_normal(5000) * 0.01,
                        g.uniform(-448, 448, 5000), [0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10]])
    x = x.astype(np.float32)
    assert np.array_equal(f8.e4m3_codes(x), torch_e4m3(x))


def test_e4m3_ties_go_to_even_and_large_values_saturate():
    # 1 + 1/16 lies halfway between 1 (mantissa 0) and 1.125 (mantissa 1): even -> 1
    # 1 + 3/16 lies halfway between 1.125 and 1.25: even -> 1.25
    # 3 * 2^-10 lies halfway between the subnormals 2^-9 and 2 * 2^-9: even -> 2 * 2^-9
    x = np.array([1 + 1 / 16, 1 + 3 / 16, 3 * 2.0 ** -10, 460.0, 1e4, -1e4], np.float32)
    assert f8.e4m3_values(f8.e4m3_codes(x)).tolist() == [1.0, 1.25, 2 * 2.0 ** -9, 448.0, 448.0, -448.0]


def test_every_e4m3_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    back = f8.e4m3_codes(f8.e4m3_values(codes).astype(np.float32))
    assert np.array_equal(back[codes != 0x80], codes[codes != 0x80])   # -0 encodes with its sign too
    assert f8.e4m3_values([0x7E])[0] == 448.0 and f8.e4m3_values([0x01])[0] == 2.0 ** -9


# ------------------------------------------------------------------ ExpCast

def test_expcast_matches_the_page_figures():
    gv = golden()
    assert (gv["byte_slope"], gv["byte_bias"], gv["beta"]) == (8.0, f8.EXPCAST_BIAS, f8.EXPCAST_BETA)
    # one doubling of the value range inside E4M3's normal range, densely
    w = np.linspace(-3.0, -2.0, 1_000_001)[:-1]              # v = 2^w, coded value v = p 2^P_SHIFT
    direct = f8.expcast_codes(8.0 * (w - f8.P_SHIFT)).astype(int)
    cast = torch_e4m3(np.exp2(w)).astype(int)
    d = direct - cast
    assert abs((d == 0).mean() * 100 - gv["match_percent"]) < 0.05
    assert np.abs(d).max() == gv["max_code_difference"]


def test_expcast_row_total_variation_stays_under_the_page_bound():
    bound = golden()["row_tv_bound_percent"] / 100
    g = np.random.default_rng(2)
    worst = 0.0
    for sigma in (0.3, 1.0, 2.0, 4.0):
        for _ in range(200):
            x = g.standard_normal(512) * sigma                   # log2-domain logits
            x -= x.max()
            ref = f8.reference_for(8.0 * x.max())
            c = f8.expcast_codes(8.0 * x - ref)
            if c.min() < 8:                                      # underflow tail: outside the bound
                continue
            p = f8.e4m3_values(c)
            tv = 0.5 * np.abs(p / p.sum() - np.exp2(x) / np.exp2(x).sum()).sum()
            worst = max(worst, tv)
    assert 0.0 < worst < bound


# ------------------------------------------------------------------ quantisation

def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_quantize_qk_scales_codes_and_error_bound():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(1, 300, 2, 128, generator=g) * 3).to(torch.bfloat16)
    x[0, 128:256, 1] = 0                                     # an all-zero block
    codes, scale = f8.quantize_qk(_bits(x))
    xf = x.float().numpy().astype(np.float64)
    val = f8.e4m3_values(codes)
    for b in range(1):
        for h in range(2):
            for blk in range(3):
                t = slice(blk * 128, min(300, blk * 128 + 128))
                amax = np.abs(xf[b, t, h]).max()
                assert scale[b, h, blk] == np.float32(np.float32(amax) / np.float32(448))
                if amax == 0:
                    assert np.all(codes[b, t, h] == 0)
                    continue
                assert np.abs(val[b, t, h]).max() == 448.0       # the absmax element takes the top code
                # |x - s v| <= s * half a quantum, quantum <= |v| / 8 (normal) or 2^-9 (subnormal)
                err = np.abs(xf[b, t, h] - scale[b, h, blk] * val[b, t, h])
                q = np.maximum(np.abs(val[b, t, h]) / 8, 2.0 ** -9)
                assert np.all(err <= scale[b, h, blk] * (q / 2 + 1e-3 * q) + 1e-30)


def test_vsmooth_demean_restore_and_constant_blocks():
    g = torch.Generator().manual_seed(4)
    v = torch.randn(1, 300, 2, 128, generator=g)
    v[0, :, 0, 5] *= 8                                       # an outlier channel
    v[0, 128:256, 1] = 0.75                                  # a constant block
    v = v.to(torch.bfloat16)
    vs = f8.vsmooth(_bits(v))
    vf = v.float().numpy().astype(np.float64)
    for h in range(2):
        for blk, (t0, t1) in enumerate(((0, 128), (128, 256), (256, 300))):
            m64 = vf[0, t0:t1, h].mean(axis=0)
            assert np.allclose(vs["mu"][0, h, blk], m64, rtol=0, atol=1e-6 * (1 + np.abs(m64)))
    assert np.all(vs["codes"][0, 128:256, 1] == 0) and np.all(vs["mu"][0, 1, 1] == np.float32(0.75))
    # restore: v ~ code * scale + mu within half a quantum of the channel scale
    rec = f8.e4m3_values(vs["codes"]) * vs["scale"][:, None] + np.repeat(vs["mu"], 128, axis=2)[:, :, :300].transpose(0, 2, 1, 3)
    q = np.maximum(np.abs(f8.e4m3_values(vs["codes"])) / 8, 2.0 ** -9) * vs["scale"][:, None]
    assert np.all(np.abs(rec - vf) <= q / 2 + 1e-6 * np.abs(vf) + 1e-7)
    # the outlier channel gets its own, larger scale
    assert vs["scale"][0, 0, 5] > 4 * np.median(vs["scale"][0, 0])
    # hi + lo carries mu / scale to about 2^-16
    mu_p = bits_to_float(vs["mu_hi"]) + bits_to_float(vs["mu_lo"])
    with np.errstate(divide="ignore", invalid="ignore"):
        want = np.where(vs["scale"][:, :, None, :] > 0, vs["mu"] / vs["scale"][:, :, None, :].astype(np.float64), 0)
    assert np.allclose(mu_p * vs["scale"][:, :, None, :], vs["mu"], rtol=2 ** -15, atol=1e-30)
    assert np.allclose(mu_p, want, rtol=2 ** -14)


# ------------------------------------------------------------------ the 8-bit attention

def _qkv(B, H, Sq, Skv, seed, scale_q=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Sq, H, 128, generator=g) * scale_q).to(torch.bfloat16)
    k = torch.randn(B, Skv, H, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Skv, H, 128, generator=g).to(torch.bfloat16)
    return q, k, v


def test_zero_query_gives_the_mean_of_the_restored_values_and_a_closed_form_lse():
    q, k, v = _qkv(1, 2, 130, 300, 5)
    q.zero_()
    o, lse = f8.attention_fp8(_bits(q), _bits(k), _bits(v), 1 / math.sqrt(128))
    vs = f8.vsmooth(_bits(v))
    rec = f8.e4m3_values(vs["codes"]) * vs["scale"][:, None] + \
        np.repeat(vs["mu"], 128, axis=2)[:, :, :300].transpose(0, 2, 1, 3)
    # every logit is 0: reference 0.65, every byte rint(95.65 - 0.65) = 95 = 1.875 * 2^4 = 30
    assert f8.reference_for(0.0) == pytest.approx(0.65)
    assert f8.e4m3_values([95])[0] == 30.0
    for h in range(2):
        assert np.allclose(o[0, :, h], rec[0, :, h].mean(axis=0), rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], math.log(2) * (0.65 / 8 - 5 + math.log2(300 * 30.0)), rtol=1e-13)


def test_constant_values_come_back_exactly():
    q, k, v = _qkv(1, 1, 200, 333, 6)
    v = torch.full_like(v, -1.375)
    o, _ = f8.attention_fp8(_bits(q), _bits(k), _bits(v), 1 / math.sqrt(128))
    assert np.allclose(o, -1.375, rtol=1e-12)


def test_a_dominant_key_selects_its_value_row():
    q, k, v = _qkv(1, 1, 4, 256, 7)
    q = torch.zeros_like(q)
    q[0, :, 0, 0] = 8.0
    k = torch.zeros_like(k)
    k[0, 200, 0, 0] = 8.0                                    # logit 64 / sqrt(128) * 8 ... far above the rest
    scale = 1.0
    o, lse = f8.attention_fp8(_bits(q), _bits(k), _bits(v), scale)
    vs = f8.vsmooth(_bits(v))
    want = f8.e4m3_values(vs["codes"][0, 200, 0]) * vs["scale"][0, 0] + vs["mu"][0, 0, 1]
    for i in range(4):
        assert np.allclose(o[0, i, 0], want, rtol=0, atol=1e-9)
        assert lse[0, 0, i] == pytest.approx(64.0, abs=0.05)


def _dequantized(q, k, v):
    """The tensors the 8-bit path multiplies, back in float64 [B, S, H, D]."""
    S, Skv = q.shape[1], k.shape[1]
    qc, qs = f8.quantize_qk(_bits(q))
    kc, ks = f8.quantize_qk(_bits(k))
    vs = f8.vsmooth(_bits(v))
    qd = f8.e4m3_values(qc) * np.repeat(qs, 128, axis=2)[:, :, :S].transpose(0, 2, 1)[..., None]
    kd = f8.e4m3_values(kc) * np.repeat(ks, 128, axis=2)[:, :, :Skv].transpose(0, 2, 1)[..., None]
    vd = f8.e4m3_values(vs["codes"]) * vs["scale"][:, None] + \
        np.repeat(vs["mu"], 128, axis=2)[:, :, :Skv].transpose(0, 2, 1, 3)
    return qd, kd, vd


def _sdpa64(q, k, v, scale, mask, chunk):
    """torch float64 attention on [B, S, H, D] arrays with the block-causal mask expanded."""
    Q, K, V = (torch.tensor(x).permute(0, 2, 1, 3) for x in (q, k, v))
    Sq, Skv = Q.shape[2], K.shape[2]
    m = None
    if mask == MASK_BLOCK_CAUSAL:
        i = torch.arange(Sq)[:, None] // chunk
        j = torch.arange(Skv)[None, :] // chunk
        m = j <= i
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m, scale=scale)
    logits = (Q @ K.transpose(-1, -2)) * scale
    if m is not None:
        logits = logits.masked_fill(~m, float("-inf"))
    return o.permute(0, 2, 1, 3).numpy(), torch.logsumexp(logits, dim=-1).numpy()


def _rel(a, b):
    return np.sqrt(((a - b) ** 2).mean()) / np.sqrt((b ** 2).mean())


@pytest.mark.parametrize("mask,chunk,sort_keys", [(MASK_FULL, 0, False), (MASK_FULL, 0, True),
                                                  (MASK_BLOCK_CAUSAL, 200, False)])
def test_fp8_attention_error_splits_into_expcast_and_quantisation(mask, chunk, sort_keys):
    B, H, S = 1, 2, 600
    q, k, v = _qkv(B, H, S, S, 8, scale_q=2.0)
    if sort_keys:
        # keys ordered so that every tile's max exceeds the last: the reference is raised again and again
        order = torch.argsort(k[0, :, :, :].float().sum(-1).mean(-1))
        k, v = k[:, order], v[:, order]
        q[0, :, :, :] = k[0, -1:, :, :].float().expand(S, H, 128).to(torch.bfloat16) * 0.5
    scale = 1 / math.sqrt(128)
    o8, l8 = f8.attention_fp8(_bits(q), _bits(k), _bits(v), scale, mask, chunk)
    # ExpCast alone: exact softmax over the same dequantized tensors differs by the
    # page's per-row total-variation scale at most
    qd, kd, vd = _dequantized(q, k, v)
    od, ld = _sdpa64(qd, kd, vd, scale, mask, chunk)
    tv = golden()["row_tv_bound_percent"] / 100
    assert _rel(o8, od) < tv
    assert np.abs(l8 - ld).max() < tv                       # ln of a sum off by under the same fraction
    # against exact attention on the bf16 inputs: the 8-bit quantisation error on top
    o, l = attention(_bits(q), _bits(k), _bits(v), scale, mask, chunk)
    assert _rel(o8, o) < 0.10
    assert (np.abs(l8 - l) / np.maximum(np.abs(l), 1)).max() < 0.03


# ------------------------------------------------------------------ the plain ExpCast statement

def test_plain_expcast_row_matches_the_page_figures():
    """Row bytes against the row's own max: in one doubling of the value range,
    79.6% equal the bytes of exp-then-cast and none is more than one code off."""
    gv = golden()
    u = np.linspace(-16.0, -8.0, 1_000_001)[:-1]          # code units below the max: values 2^3 .. 2^4
    z = np.concatenate([[0.0], u]) + 123.25               # any offset: only z - max z matters
    bytes_ = f8.expcast_row(z).astype(int)[1:]
    cast = torch_e4m3(np.exp2(u / 8.0 + f8.P_SHIFT)).astype(int)
    d = bytes_ - cast
    assert abs((d == 0).mean() * 100 - gv["match_percent"]) < 0.05
    assert np.abs(d).max() == gv["max_code_difference"]
    assert f8.expcast_row(np.array([3.0, 3.0, -np.inf]))[:2].tolist() == [96, 96]   # the max: 2^P_SHIFT
    assert f8.expcast_row(np.array([0.0, -np.inf]))[1] == 0


def test_plain_expcast_row_total_variation_stays_under_the_page_bound():
    bound = golden()["row_tv_bound_percent"] / 100
    g = np.random.default_rng(12)
    worst = 0.0
    for sigma in (0.3, 1.0, 2.0):
        for _ in range(200):
            x = g.standard_normal(700) * sigma               # log2-domain logits
            c = f8.expcast_row(8.0 * x)
            if c.min() < 8:                                  # underflow tail: outside the bound
                continue
            p = f8.e4m3_values(c)
            e = np.exp2(x - x.max())
            tv = 0.5 * np.abs(p / p.sum() - e / e.sum()).sum()
            worst = max(worst, tv)
    assert 0.0 < worst < bound


def test_log_error_spread_of_the_byte_map():
    """SIGMA_LN_R (tests/helpers.py): the standard deviation of
    ln value(rint(u + 95.65)) - (u/8 + 5) ln 2 over the normal codes, and the
    range of that log error (half a code plus the mantissa's linear
    approximation of 2^x, about 7% either way)."""
    from tests.helpers import SIGMA_LN_R
    u = np.linspace(-56.0, 0.0, 4_000_001)
    c = f8.expcast_codes(u)
    assert c.min() >= 8                                      # all normal
    lnr = np.log(f8.e4m3_values(c)) - (u / 8 + f8.P_SHIFT) * math.log(2)
    assert abs(lnr.std() - SIGMA_LN_R) < 5e-4
    assert np.abs(lnr).max() < 0.075
    assert abs(lnr.mean()) < 0.01                            # beta centres it


def test_plain_closed_forms():
    scale = 1 / math.sqrt(128)
    # Q = 0: every byte is 96 (value 2^5), so O is the mean of V-Smooth's
    # reconstruction and LSE = ln n exactly
    q, k, v = _qkv(1, 2, 130, 300, 15)
    q.zero_()
    o, lse = f8.attention_fp8_plain(_bits(q), _bits(k), _bits(v), scale)
    _, _, vd = _dequantized(q, k, v)
    for h in range(2):
        assert np.allclose(o[0, :, h], vd[0, :, h].mean(axis=0), rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], math.log(300), rtol=0, atol=1e-12)
    # block-causal Q = 0: the mean over the allowed prefix, LSE = ln |A(i)|
    o, lse = f8.attention_fp8_plain(_bits(q), _bits(k[:, :130]), _bits(v[:, :130]), scale, MASK_BLOCK_CAUSAL, 50)
    _, _, vd = _dequantized(q, k[:, :130], v[:, :130])
    for i in (0, 49, 50, 129):
        n = min(130, (i // 50 + 1) * 50)
        assert np.allclose(o[0, i, 1], vd[0, :n, 1].mean(axis=0), rtol=0, atol=1e-12)
        assert lse[0, 1, i] == pytest.approx(math.log(n), abs=1e-12)
    # constant V comes back exactly
    q, k, v = _qkv(1, 1, 200, 333, 16)
    v = torch.full_like(v, 0.625)
    o, _ = f8.attention_fp8_plain(_bits(q), _bits(k), _bits(v), scale)
    assert np.allclose(o, 0.625, rtol=1e-12)
    # one dominant key selects its reconstructed value row; LSE is its logit
    q, k, v = _qkv(1, 1, 4, 256, 17)
    q = torch.zeros_like(q)
    q[0, :, 0, 0] = 8.0
    k = torch.zeros_like(k)
    k[0, 200, 0, 0] = 8.0
    o, lse = f8.attention_fp8_plain(_bits(q), _bits(k), _bits(v), 1.0)
    _, _, vd = _dequantized(q, k, v)
    for i in range(4):
        assert np.allclose(o[0, i, 0], vd[0, 200, 0], rtol=0, atol=1e-9)
        assert lse[0, 0, i] == pytest.approx(64.0, abs=0.05)


def test_plain_statement_is_close_to_exact_softmax_on_the_same_operands():
    """Only ExpCast separates the plain statement from exact attention on the
    dequantised tensors: within the page's per-row total-variation scale."""
    q, k, v = _qkv(1, 2, 600, 600, 18, scale_q=2.0)
    scale = 1 / math.sqrt(128)
    o8, l8 = f8.attention_fp8_plain(_bits(q), _bits(k), _bits(v), scale)
    qd, kd, vd = _dequantized(q, k, v)
    od, ld = _sdpa64(qd, kd, vd, scale, MASK_FULL, 0)
    tv = golden()["row_tv_bound_percent"] / 100
    assert _rel(o8, od) < tv
    assert np.abs(l8 - ld).max() < tv


@pytest.mark.parametrize("mask,chunk,sort_keys", [(MASK_FULL, 0, False), (MASK_FULL, 0, True),
                                                  (MASK_BLOCK_CAUSAL, 300, False)])
def test_tiled_schedule_stays_within_the_derived_bound_of_the_plain_statement(mask, chunk, sort_keys):
    """The schedule the kernel uses (attention_fp8: 128-key tiles, lazily raised
    reference on a grid) against the plain statement, under the bars the GPU
    test applies to the kernel (tests/helpers.py); zeros, a 10% gain and
    shuffled rows must fail those bars."""
    from tests.helpers import check_expcast_parity
    B, H, S = 1, 2, 1000
    q, k, v = _qkv(B, H, S, S, 19, scale_q=1.5)
    if sort_keys:
        order = torch.argsort(k[0].float().sum(-1).mean(-1))   # every tile raises the reference
        k, v = k[:, order], v[:, order]
    scale = 1 / math.sqrt(128)
    quant = (f8.quantize_qk(_bits(q)), f8.quantize_qk(_bits(k)), f8.vsmooth(_bits(v)))
    o_t, l_t = f8.attention_fp8(None, None, None, scale, mask, chunk, quantized=quant)
    o_p, l_p, s_o, s_l = f8.attention_fp8_plain(None, None, None, scale, mask, chunk, quantized=quant, spread=True)
    flat = lambda a: np.concatenate([a[0, :, h] for h in range(H)])      # noqa: E731
    flat_l = lambda a: np.concatenate([a[0, h] for h in range(H)])       # noqa: E731
    groups = [np.arange(i * S, (i + 1) * S) for i in range(H)]
    res = check_expcast_parity(flat(o_t), flat(o_p), flat_l(l_t), flat_l(l_p), flat(s_o), flat_l(s_l), groups)
    assert res["ok"], res
    assert res["rel_rms"] < 0.06
    for bad in (np.zeros_like(o_t), 1.1 * o_t, o_t[:, np.random.default_rng(0).permutation(S)]):
        assert not check_expcast_parity(flat(bad), flat(o_p), None, None, flat(s_o), None, groups)["ok"]
