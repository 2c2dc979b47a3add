"""The parity checker must reject outputs that carry no information."""
import numpy as np

from tests.helpers import check_parity, round_bf16


def test_checker_accepts_the_reference_and_rejects_zeros_and_shuffles():
    rng = np.random.default_rng(0)
    n, D, S = 512, 128, 75600
    o_ref = rng.standard_normal((n, D)) * np.sqrt(np.e / S)  # attention-sized outputs
    lse = 11.0 + rng.standard_normal(n) * 0.1
    assert check_parity(round_bf16(o_ref), o_ref, lse, lse)["ok"]
    zeros = check_parity(np.zeros_like(o_ref), o_ref, lse, lse)
    assert not zeros["ok"]
    shuffled = round_bf16(o_ref[rng.permutation(n)])
    assert not check_parity(shuffled, o_ref, lse, lse)["ok"]
    assert not check_parity(round_bf16(o_ref), o_ref, lse + 0.05, lse)["ok"]


def test_excess_over_rounding_bar():
    """The output's own bf16 rounding passes the excess bar, also in channels
    eight times larger than the rest and in channels that barely vary; an
    error of 3% of the head's rms beyond that rounding fails it."""
    from tests.helpers import EXCESS_BAR
    rng = np.random.default_rng(1)
    n, D, S = 512, 128, 32760
    o_ref = rng.standard_normal((n, D)) * np.sqrt(np.e / S)
    o_ref[:, [5, 77, 100]] *= 8.0                       # value-outlier channels
    o_ref[:, 3] = 1e-6 + 1e-9 * rng.standard_normal(n)  # a channel that barely varies
    lse = 10.0 + rng.standard_normal(n) * 0.1
    res = check_parity(round_bf16(o_ref), o_ref, lse, lse)
    assert res["ok"] and res["max_excess_over_channel_rms"] <= EXCESS_BAR, res
    rms = np.sqrt(np.mean(o_ref ** 2))
    bad = round_bf16(o_ref)
    bad[17, 40] += 0.03 * rms + 2.0 ** -7 * abs(o_ref[17, 40])
    res = check_parity(bad, o_ref, lse, lse)
    assert not res["ok"] and res["max_excess_over_channel_rms"] > EXCESS_BAR
    assert check_parity(bad, o_ref, lse, lse, excess_bar=None)["ok"]
