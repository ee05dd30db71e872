"""CPU checks behind the activation-range parity tests.

1. The cases of tests/test_gpu_activation_range.py discriminate: rounding the activations
   to 31-bit fixed point relative to the largest |x| of each block of 1024 k (what a
   fixed-point tensor-core GEMV would do) breaks the qgemm tolerance
   |dy| <= 1e-5 * sum_k |w'x| + 1e-6 there, so a GPU path that passed them cannot be
   rounding that way.
2. The exact split that the GEMV uses instead: every fp32 x is hi + mid + lo with three
   bf16 values (hi = x with the low 16 bits of its encoding cleared, mid the same of
   x - hi, lo = x - hi - mid), so the tensor-core products code * piece are exact and the
   only roundings left are those of fp32 sums.
"""
import numpy as np
import pytest

import oracle

RTOL, ATOL = 1e-5, 1e-6


def bf16_trunc(v: np.ndarray) -> np.ndarray:
    return (v.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def split3(x: np.ndarray):
    x = x.astype(np.float32)
    hi = bf16_trunc(x)
    r = (x - hi).astype(np.float32)
    mid = bf16_trunc(r)
    lo = (r - mid).astype(np.float32)
    return hi, mid, lo


def is_bf16(v: np.ndarray) -> bool:
    return bool(np.all((v.view(np.uint32) & np.uint32(0xFFFF)) == 0))


def block_fixed_point(x: np.ndarray, block: int = 1024, bits: int = 30) -> np.ndarray:
    """x rounded to multiples of 2^(E - bits), max |x| of each block of k below 2^E."""
    out = np.empty_like(x, dtype=np.float64)
    for m in range(x.shape[0]):
        for b0 in range(0, x.shape[1], block):
            blk = x[m, b0:b0 + block].astype(np.float64)
            mx = np.abs(blk).max()
            if mx == 0:
                out[m, b0:b0 + block] = 0
                continue
            E = int(np.floor(np.log2(mx))) + 1
            q = 2.0 ** (E - bits)
            out[m, b0:b0 + block] = np.rint(blk / q) * q
    return out


def fraction_outside(w, x, bits, group, xq):
    N, K = w.shape
    payload, scales, _ = oracle.pack(w, bits, group)
    yref, bound = oracle.qgemm(x, payload, scales, N, K, bits, group)
    wq = oracle.dequant_rows(payload, scales, N, K, bits, group).astype(np.float64)
    y_fixed = xq @ wq.T
    return float(np.mean(np.abs(y_fixed - yref) > RTOL * bound + ATOL))


def test_huge_activation_on_zero_code_column_breaks_fixed_point():
    rng = np.random.default_rng(0)
    N, K = 256, 1024
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w[rng.random(N) < 0.9, 137] = 0.0
    x = rng.normal(0, 1, (1, K)).astype(np.float32)
    x[0, 137] = 1e7
    assert fraction_outside(w, x, 4, 128, block_fixed_point(x)) > 0.5
    # the exact split keeps every row inside the bound (the products are exact)
    hi, mid, lo = split3(x)
    xs = hi.astype(np.float64) + mid + lo
    assert np.array_equal(xs, x.astype(np.float64))
    assert fraction_outside(w, x, 4, 128, xs) == 0.0


def test_small_activations_with_one_large_break_fixed_point():
    rng = np.random.default_rng(1)
    N, K = 256, 1024
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w[rng.random(N) < 0.95, 500] = 0.0
    x = rng.normal(0, 1e-3, (1, K)).astype(np.float32)
    x[0, 500] = 1e4
    assert fraction_outside(w, x, 8, 128, block_fixed_point(x)) > 0.5


@pytest.mark.parametrize("scale", [1e-30, 1e-8, 1.0, 1e8, 1e30])
def test_split3_is_exact(scale):
    rng = np.random.default_rng(7)
    x = (rng.normal(0, 1, 100000) * scale).astype(np.float32)
    x = x[np.abs(x) >= 2.0 ** -110]  # below that, see the next tests
    hi, mid, lo = split3(x)
    assert is_bf16(hi) and is_bf16(mid) and is_bf16(lo)
    assert np.array_equal(hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64),
                          x.astype(np.float64))
    # products with any code |c| <= 127 stay exact in fp32 (8 + 8 significant bits)
    for p in (hi, mid, lo):
        c = rng.integers(-127, 128, p.size).astype(np.float32)
        assert np.array_equal((c * p).astype(np.float64), c.astype(np.float64) * p.astype(np.float64))


def test_split3_extremes():
    vals = np.array([0.0, -0.0, 1.0, -1.0, np.finfo(np.float32).max, -np.finfo(np.float32).max,
                     np.finfo(np.float32).tiny, 2.0 ** -110, 1.0 + 2.0 ** -23, 3.4e38, 1e-38],
                    dtype=np.float32)
    hi, mid, lo = split3(vals)
    assert np.array_equal(hi.astype(np.float64) + mid + lo, vals.astype(np.float64))


def test_split3_below_2_to_minus_110_loses_under_2_to_minus_126():
    # the last piece can lose bits only for |x| < 2^-110; the loss stays below 2^-126
    rng = np.random.default_rng(3)
    x = (rng.random(100000) * 2.0 ** -110).astype(np.float32)
    hi, mid, lo = split3(x)
    lo_b = bf16_trunc(lo)  # what the bf16 column holds
    err = np.abs(hi.astype(np.float64) + mid + lo_b - x.astype(np.float64))
    assert err.max() < 2.0 ** -126
