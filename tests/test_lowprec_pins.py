"""Pins of the oracle's bf16 rounding (low-precision compressed keys).

"CSA + HCA 混合注意力机制" §4.2 runs the indexer's QK path at reduced precision;
here the compressed keys may be stored as bf16.  The oracle rounds its
float64 mean to the nearest bf16 value (ties to even) in one step.  Pins: on
binary32 inputs (where one rounding from binary32 is the whole story) it
agrees with torch's binary32 -> bf16 conversion; on binary64 inputs the
result is a bf16 value no farther from x than either neighbour, ties even,
checked in exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _bf16_bits(x: float) -> int:
    return int(np.float32(x).view(np.uint32)) >> 16


def _bf16_value(bits: int) -> float:
    return float(np.uint32(bits << 16).view(np.float32))


def test_round_bf16_matches_torch_on_binary32_values():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)
    # exact ties: halfway between two bf16 values, both parities
    ties = np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -(1.0 + 2.0**-8), 2.0**-130 + 2.0**-134], np.float32)
    assert np.array_equal(oracle.round_bf16(ties.astype(np.float64)),
                          torch.from_numpy(ties).to(torch.bfloat16).double().numpy())


@pytest.mark.parametrize("seed", range(5))
def test_round_bf16_is_nearest_ties_even_on_binary64(seed):
    rng = np.random.default_rng(100 + seed)
    x = rng.normal(size=400) * np.exp2(rng.integers(-140, 120, size=400))
    y = oracle.round_bf16(x)
    for xi, yi in zip(x.tolist(), y.tolist()):
        b = _bf16_bits(yi)
        assert _bf16_value(b) == yi, "not a bf16 value"
        fx, fy = Fraction(xi), Fraction(yi)
        for nb in (b - 1, b + 1):
            if nb & 0x7f80 == 0x7f80 or nb < 0:      # skip inf/NaN codes
                continue
            v = _bf16_value(nb)
            if np.sign(v) != np.sign(yi) and v != 0:
                continue
            d_other, d_mine = abs(Fraction(v) - fx), abs(fy - fx)
            assert d_mine <= d_other
            if d_mine == d_other:
                assert b % 2 == 0, "tie not to even"


def test_round_bf16_special_values():
    assert oracle.round_bf16(0.0) == 0.0
    assert np.isinf(oracle.round_bf16(3.5e38))                    # above the largest finite bf16
    big = _bf16_value(0x7f7f)                                      # largest finite
    assert oracle.round_bf16(big) == big and oracle.round_bf16(big * (1 + 2.0**-10)) == big
    assert np.isnan(oracle.round_bf16(float("nan")))
