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
