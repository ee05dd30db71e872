"""GPTQ as the pages define it -- TEST INFRASTRUCTURE ONLY (the oracle).

Only the tests may import this module. It follows "Huit bits, puis quatre", section
"Arrondir mieux : GPTQ": the inputs of a layer enter through H = sum over samples of
x^T x ([K, K]); a damping of 1 % of the mean of H's diagonal is added; H^-1 = U^T U with
U upper triangular (the Cholesky factor of the inverse). The input components k (the
columns of our W [N, K], the rows of the page's W) are quantized one after another:

    q_k    = round(w_k)                       (the group's grid, below)
    error  = (w_k - q_k) / U[k, k]
    w_j   -= error * U[k, j]                  for every j > k

and a group's scales are fixed when its first column is reached, from the weights
corrected so far. The grid and the rounding are those of the "Arrondir" rule (scale =
max|w| / qmax in fp32, a zero scale becomes 1, code = clip(rint(w / scale)) with an fp32
divide), applied to the corrected weights rounded to fp32; everything else is fp64.

Reading where the page is silent: the quantity subtracted is the weight minus its
dequantized value code * scale (q_k above is that value); the stored format is the one
of pack(): one scale per g consecutive weights along K, int4 codes + 8 two per byte with
the even element in the low nibble.

numpy.linalg's inverse and Cholesky factorisation serve as library steps.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

QMAX = {4: 7, 8: 127}


def damped(H: np.ndarray, damp: float = 0.01) -> np.ndarray:
    """H + damp * mean(diag(H)) * I, in fp64."""
    H = np.array(H, dtype=np.float64)
    K = H.shape[0]
    return H + damp * float(np.mean(np.diag(H))) * np.eye(K)


def hinv_chol_upper(H: np.ndarray, damp: float = 0.01) -> np.ndarray:
    """U, upper triangular, with (H + damping)^-1 = U^T U."""
    Hinv = np.linalg.inv(damped(H, damp))
    Hinv = (Hinv + Hinv.T) / 2.0  # the inverse of a symmetric matrix, symmetric to the last bit
    return np.linalg.cholesky(Hinv).T  # lower L with L L^T = Hinv, so U = L^T


def _group_scales(block: np.ndarray, bits: int) -> np.ndarray:
    """Scales of one group for every row, from its current weights (fp32 rule)."""
    a = np.max(np.abs(block.astype(np.float32)), axis=1)
    s = (a / np.float32(QMAX[bits])).astype(np.float32)
    s[s == 0] = np.float32(1.0)
    return s


def gptq_codes(w: np.ndarray, U: np.ndarray, bits: int, group: int) -> Tuple[np.ndarray, np.ndarray]:
    """Codes int8 [N, K] and scales float32 [N, K/group] of W [N, K] given U."""
    W = np.array(w, dtype=np.float64)  # the weights being corrected
    N, K = W.shape
    if group < 1 or K % group:
        raise ValueError("group must divide K")
    qmax = QMAX[bits]
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // group), np.float32)
    s = None
    for k in range(K):
        if k % group == 0:
            s = _group_scales(W[:, k:k + group], bits)
            scales[:, k // group] = s
        t = W[:, k].astype(np.float32) / s
        c = np.clip(np.rint(t), -qmax, qmax).astype(np.int8)
        codes[:, k] = c
        wq = (c.astype(np.float32) * s).astype(np.float64)  # code * scale, exact in fp32
        err = (W[:, k] - wq) / U[k, k]
        W[:, k + 1:] -= np.outer(err, U[k, k + 1:])
    return codes, scales


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """The payload bytes of codes, flattened row-major as pack() stores them."""
    c = np.ascontiguousarray(codes, dtype=np.int8).reshape(-1)
    if bits == 8:
        return c.view(np.uint8).copy()
    u = (c.astype(np.int16) + 8).astype(np.uint8)
    return (u[0::2] | (u[1::2] << 4)).astype(np.uint8)


def gptq(w: np.ndarray, H: np.ndarray, bits: int, group: int, damp: float = 0.01):
    """(payload, scales flat, codes [N, K], U) of W [N, K] for inputs with H = sum x^T x."""
    U = hinv_chol_upper(H, damp)
    codes, scales = gptq_codes(w, U, bits, group)
    return pack_codes(codes, bits), scales.reshape(-1), codes, U


def dequant(codes: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """code * scale in fp32, [N, K]."""
    N, K = codes.shape
    s = np.repeat(np.asarray(scales, np.float32).reshape(N, K // group), group, axis=1)
    return (codes.astype(np.float32) * s).astype(np.float32)
