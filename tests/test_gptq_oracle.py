"""Pins for the GPTQ oracle ("Huit bits, puis quatre", section "Arrondir mieux : GPTQ").

The page states two tests of the algorithm: with independent inputs H is diagonal and GPTQ
must give exactly round-to-nearest; with correlated inputs the error of the layer's output
must drop, by more than 30 % on a synthetic example. A third pin computes the same greedy
quantizer from its original definition (Frantar et al., 2022, the OBS update with the
inverse of the Hessian restricted to the columns not yet quantized, taken afresh at every
step), which the page's Cholesky form reorganises: the codes must agree.
"""
import numpy as np
import pytest

import oracle
from oracle import gptq as G

QMAX = {4: 7, 8: 127}


def correlated_inputs(S, K, rank, seed, noise=0.05):
    """x = z A + noise: K input components driven by `rank` shared factors."""
    rng = np.random.default_rng(seed)
    z = rng.normal(0, 1, (S, rank))
    A = rng.normal(0, 1, (rank, K))
    return (z @ A + noise * rng.normal(0, 1, (S, K))).astype(np.float64)


def output_err(X, w, wq):
    d = X @ (np.asarray(w, np.float64) - np.asarray(wq, np.float64)).T
    return float(np.sum(d * d))


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (8, 64), (4, 256), (8, 256)])
def test_diagonal_hessian_gives_round_to_nearest(bits, group):
    # independent inputs: H diagonal, nothing to compensate -> the RTN codes and scales
    rng = np.random.default_rng(bits + group)
    N, K = 24, 256
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w.reshape(-1)[rng.choice(N * K, 20, replace=False)] *= 20
    H = np.diag(rng.uniform(0.5, 3.0, K))
    payload, scales, _, U = G.gptq(w, H, bits, group)
    assert np.count_nonzero(np.triu(U, 1)) == 0
    rp, rs, st = oracle.pack(w, bits, group)
    assert st == oracle.OK
    assert np.array_equal(payload, rp)
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("bits,group", [(4, 256), (4, 32), (8, 256)])
def test_correlated_inputs_lower_the_output_error_by_more_than_30_percent(bits, group):
    S, N, K = 4096, 64, 256
    X = correlated_inputs(S, K, rank=16, seed=7 + bits)
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    _, scales, codes, _ = G.gptq(w, X.T @ X, bits, group)
    wg = G.dequant(codes, scales, group)
    rp, rs, _ = oracle.pack(w, bits, group)
    wr = oracle.dequant(rp, rs, N * K, bits, group).reshape(N, K)
    e_rtn, e_gptq = output_err(X, w, wr), output_err(X, w, wg)
    assert e_gptq < 0.7 * e_rtn, (e_gptq / e_rtn)


def obs_reference(w, H, bits, group, damp=0.01):
    """The greedy OBS quantizer with explicit inverses (O(K^4); tiny K only)."""
    W = np.array(w, np.float64)
    N, K = W.shape
    Hd = np.array(H, np.float64) + damp * np.mean(np.diag(H)) * np.eye(K)
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // group), np.float32)
    for k in range(K):
        if k % group == 0:
            a = np.max(np.abs(W[:, k:k + group].astype(np.float32)), axis=1)
            s = (a / np.float32(QMAX[bits])).astype(np.float32)
            s[s == 0] = 1
            scales[:, k // group] = s
        c = np.clip(np.rint(W[:, k].astype(np.float32) / s), -QMAX[bits], QMAX[bits])
        codes[:, k] = c
        q = (c.astype(np.float32) * s).astype(np.float64)
        F = np.arange(k, K)  # columns not yet fixed, k first
        Finv = np.linalg.inv(Hd[np.ix_(F, F)])
        # optimal change of the free weights once w_k is pinned to q:
        # delta_F = -(w_k - q) / [H_F^-1]_kk * [H_F^-1]_{k, F}
        W[:, F] -= np.outer((W[:, k] - q) / Finv[0, 0], Finv[0, :])
    return codes, scales


@pytest.mark.parametrize("K,group,seed", [(8, 8, 0), (16, 8, 1), (24, 8, 2), (16, 16, 3)])
@pytest.mark.parametrize("bits", [4, 8])
def test_matches_the_obs_update_with_explicit_inverses(K, group, seed, bits):
    N = 40
    X = correlated_inputs(512, K, rank=3, seed=seed)
    rng = np.random.default_rng(seed + 10)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    H = X.T @ X
    _, scales, codes, _ = G.gptq(w, H, bits, group)
    rc, rs = obs_reference(w, H, bits, group)
    assert np.array_equal(codes, rc)
    assert np.array_equal(scales.reshape(N, -1), rs)


def test_invariants_and_zero_matrix():
    rng = np.random.default_rng(5)
    N, K = 16, 64
    X = correlated_inputs(256, K, rank=4, seed=5)
    w = rng.normal(0, 0.05, (N, K)).astype(np.float32)
    for bits in (4, 8):
        _, scales, codes, _ = G.gptq(w, X.T @ X, bits, 32)
        assert np.all(np.abs(codes) <= QMAX[bits]) and np.all(scales > 0)
        # the first column of every group is quantized before any compensation reaches it
        # from its own group; the absmax of the corrected group sets an extremal code or smaller
        assert np.all(np.abs(codes).reshape(N, -1, 32).max(axis=2) <= QMAX[bits])
    payload, scales, codes, _ = G.gptq(np.zeros((4, 64), np.float32), X.T @ X, 4, 32)
    assert np.all(scales == 1) and np.all(codes == 0) and np.all(payload == 0x88)


def test_hinv_factor():
    X = correlated_inputs(300, 48, rank=6, seed=9)
    H = X.T @ X
    U = G.hinv_chol_upper(H)
    assert np.allclose(np.tril(U, -1), 0)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(48)
    assert np.allclose(U.T @ U @ Hd, np.eye(48), atol=1e-8)
