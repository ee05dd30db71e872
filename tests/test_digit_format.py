"""CPU checks of the integer-digit format the one-row GEMV uses for stages whose
activations span at most 2^21 (the other stages take the exact bf16 pieces).

For such a stage, with max |x| < 2^E, every activation becomes X = rint(x * 2^(38 - E)),
|X| < 2^38, written as five balanced base-256 digits in [-128, 127]. The digits must
reproduce X exactly, and the rounding of x must stay within 2^-18 of every nonzero |x|
(the range condition makes that hold), which keeps each product inside the qgemm bound
|dy| <= 1e-5 * sum_k |w'x| + 1e-6 with room for the fp32 sums.
"""
import numpy as np
import pytest


def exp_above(mx):
    return int(np.floor(np.log2(mx))) + 1


def digits5(x, E):
    X = np.rint(x.astype(np.float64) * 2.0 ** (38 - E)).astype(np.int64)
    U = (X + 0x8080808080) ^ 0x8080808080
    d = [((U >> (8 * p)) & 0xFF).astype(np.int64) for p in range(5)]
    d = [np.where(v >= 128, v - 256, v) for v in d]
    return X, d


@pytest.mark.parametrize("seed", range(5))
def test_digits_reconstruct_exactly_and_bound_the_rounding(seed):
    rng = np.random.default_rng(seed)
    x = (rng.normal(0, 1, 4096) * 10.0 ** rng.uniform(-5, 5)).astype(np.float32)
    mx = float(np.abs(x).max())
    E = exp_above(mx)
    keep = np.abs(x) >= 2.0 ** (E - 21)
    x = x[keep]
    X, d = digits5(x, E)
    assert np.all(np.abs(X) < 2 ** 38)
    assert all(np.all((v >= -128) & (v <= 127)) for v in d)
    assert np.array_equal(sum(v * 256 ** p for p, v in enumerate(d)), X)
    rel = np.abs(X * 2.0 ** (E - 38) - x.astype(np.float64)) / np.abs(x.astype(np.float64))
    assert rel.max() <= 2.0 ** -18


def test_digit_group_sums_fit_int32():
    # worst case of one flush: 256 k (a whole int4 stage) of |16 * code| <= 112 against
    # digits of magnitude 128, and a column pair combined as 256 * c0 + c1
    worst = 256 * 112 * 128
    assert worst < 2 ** 31 and 256 * worst + worst < 2 ** 31
