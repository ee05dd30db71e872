"""Exact-arithmetic helpers for pinning the oracle to mathematics, not to itself.

Everything here works on Python Fractions: the fp32 value nearest to an exact
rational (ties to even), the exact dot product, and a brute-force search for
the nearest integer code. None of it calls the oracle or the CUDA library.
"""
from fractions import Fraction

import numpy as np


def f32_bits(v) -> int:
    return int(np.array(v, np.float32).view(np.uint32))


def rn32(q: Fraction) -> np.float32:
    """The fp32 number nearest to the rational q, ties to even significand."""
    approx = np.float32(float(q))  # within an ulp or two of the answer
    cands = {approx, np.nextafter(approx, np.float32(np.inf)), np.nextafter(approx, np.float32(-np.inf))}
    cands = [c for c in cands if np.isfinite(c)]
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - q)
        key = (d, f32_bits(c) & 1)  # smaller distance first, then even significand
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def nearest_code(t: np.float32, qmax: int) -> int:
    """Brute force over every code in [-qmax, qmax]: the one nearest to t, ties to even."""
    tf = Fraction(float(t))
    best = None
    for c in range(-qmax, qmax + 1):
        key = (abs(tf - c), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def exact_dot(w_row, x_row) -> Fraction:
    return sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(w_row, x_row)), Fraction(0))
