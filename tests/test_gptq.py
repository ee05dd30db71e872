"""The GPTQ host quantizer of libq4 (C++, fp64) against the GPTQ oracle.

U is compared within a relative 1e-9 (two different factorisations in fp64). Given the
same U -- the oracle's, as an input -- the codes and scales are decided by the same fp32 and
fp64 operations in the same order on both sides, so payload and scales must be identical
bit for bit. Host code: these tests run without a GPU, except the last, which reads a GPTQ
payload with the GPU kernels.
"""
import numpy as np
import pytest

import oracle
from oracle import gptq as G


@pytest.fixture(scope="module")
def q4():
    import int4_quantized_b200 as m

    m.lib()
    return m


def correlated(S, K, rank, seed):
    rng = np.random.default_rng(seed)
    return (rng.normal(0, 1, (S, rank)) @ rng.normal(0, 1, (rank, K)) + 0.05 * rng.normal(0, 1, (S, K))
            ).astype(np.float32)


@pytest.mark.parametrize("K", [1, 2, 7, 64, 200])
def test_prepare_matches_oracle(q4, K):
    X = correlated(max(4 * K, 16), K, max(1, K // 8), K)
    H = X.astype(np.float64).T @ X.astype(np.float64)
    U = q4.gptq_prepare(H)
    Uo = G.hinv_chol_upper(H)
    assert np.all(np.tril(U, -1) == 0)
    assert np.max(np.abs(U - Uo)) <= 1e-9 * np.max(np.abs(Uo))


@pytest.mark.parametrize("K", [130, 515])
def test_prepare_is_the_same_for_any_thread_count(q4, K):
    X = correlated(2 * K, K, K // 8, K + 1)
    H = X.astype(np.float64).T @ X.astype(np.float64)
    U1 = q4.gptq_prepare(H, threads=1)
    for t in (2, 3, 8):
        assert np.array_equal(q4.gptq_prepare(H, threads=t), U1)
    Uo = G.hinv_chol_upper(H)
    assert np.max(np.abs(U1 - Uo)) <= 1e-9 * np.max(np.abs(Uo))


def test_hessian_accumulates_in_fp64(q4):
    X = correlated(300, 48, 5, 1)
    H = q4.gptq_hessian(X[:100], threads=3)
    q4.gptq_hessian(X[100:], H, threads=1)
    ref = X.astype(np.float64).T @ X.astype(np.float64)
    assert np.allclose(H, ref, rtol=1e-12, atol=1e-9)
    assert np.array_equal(H, H.T)


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 128), (8, 64), (8, 256), (4, 256)])
@pytest.mark.parametrize("threads", [1, 4])
def test_quantize_bit_exact_with_the_oracles_U(q4, bits, group, threads):
    N, K = 37, 256
    X = correlated(1024, K, 12, bits + group)
    rng = np.random.default_rng(group)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w.reshape(-1)[rng.choice(N * K, 30, replace=False)] *= 20
    payload_o, scales_o, _, U = G.gptq(w, X.astype(np.float64).T @ X.astype(np.float64), bits, group)
    payload, scales = q4.gptq_quantize(w, U, bits, group, threads=threads)
    assert np.array_equal(payload, payload_o)
    assert np.array_equal(scales.view(np.uint32), scales_o.view(np.uint32))


def test_diagonal_U_is_round_to_nearest(q4):
    rng = np.random.default_rng(8)
    N, K = 20, 512
    w = rng.normal(0, 0.05, (N, K)).astype(np.float32)
    U = q4.gptq_prepare(np.diag(rng.uniform(1, 2, K)))
    for bits, g in ((4, 32), (8, 512), (4, 128)):
        payload, scales = q4.gptq_quantize(w, U, bits, g)
        rp, rs, _ = oracle.pack(w, bits, g)
        assert np.array_equal(payload, rp) and np.array_equal(scales.view(np.uint32), rs.view(np.uint32))


def test_end_to_end_lowers_output_error(q4):
    S, N, K = 4096, 48, 256
    X = correlated(S, K, 16, 21)
    w = np.random.default_rng(2).normal(0, 0.02, (N, K)).astype(np.float32)
    payload, scales = q4.gptq_pack(w, X, 4, 64)
    wg = oracle.dequant(payload, scales, N * K, 4, 64).reshape(N, K)
    rp, rs, _ = oracle.pack(w, 4, 64)
    wr = oracle.dequant(rp, rs, N * K, 4, 64).reshape(N, K)
    X64 = X.astype(np.float64)
    e = lambda wq: float(np.sum((X64 @ (w.astype(np.float64) - wq).T) ** 2))  # noqa: E731
    assert e(wg) < 0.7 * e(wr)


def test_errors(q4):
    lib = q4.lib()
    U = np.eye(8)
    w = np.zeros((2, 8), np.float32)
    with pytest.raises(q4.Q4Error):
        q4.gptq_quantize(w, U, 4, 3)  # group does not divide K
    with pytest.raises(q4.Q4Error):
        q4.gptq_quantize(w, U, 5, 8)
    with pytest.raises(q4.Q4Error):
        q4.gptq_prepare(np.zeros((4, 4)))  # mean of the diagonal is 0
    with pytest.raises(q4.Q4Error):
        q4.gptq_prepare(-np.eye(4))
    bad = w.copy()
    bad[1, 3] = np.nan
    with pytest.raises(q4.Q4Error) as e:
        q4.gptq_quantize(bad, U, 8, 8)
    assert e.value.code == q4.Q4_ERR_NONFINITE
    with pytest.raises(q4.Q4Error) as e:
        q4.gptq_hessian(np.array([[1.0, np.inf]], np.float32))
    assert e.value.code == q4.Q4_ERR_NONFINITE
    assert lib.q4_gptq_quantize(None, 0, 8, None, 4, 8, None, None, 0) == q4.Q4_OK  # N = 0: nothing to do


def test_ill_conditioned_U_reports_nonfinite_and_leaves_outputs(q4):
    # a tiny diagonal with large off-diagonal entries makes the error feedback grow past the
    # fp32 range: the call reports it and writes neither payload nor scales
    import ctypes

    K, N = 64, 4
    U = np.triu(np.full((K, K), 1e30))
    np.fill_diagonal(U, 1e-30)
    w = np.random.default_rng(0).normal(0, 1, (N, K)).astype(np.float32)
    payload = np.full(N * K // 2, 0xAB, np.uint8)
    scales = np.full(N * K // 32, -7.0, np.float32)
    vp = ctypes.c_void_p
    st = q4.lib().q4_gptq_quantize(w.ctypes.data_as(vp), N, K, U.ctypes.data_as(vp), 4, 32,
                                   payload.ctypes.data_as(vp), scales.ctypes.data_as(vp), 2)
    assert st == q4.Q4_ERR_NONFINITE
    assert np.all(payload == 0xAB) and np.all(scales == -7.0)


@pytest.mark.gpu
@pytest.mark.parametrize("bits,group", [(4, 128), (8, 512)])
def test_gptq_payload_runs_through_qgemm(q4, bits, group):
    # the same format: qdequant is bit-exact and qgemm is within tolerance of the oracle
    import torch

    N, K = 300, 1024
    X = correlated(2048, K, 32, 5)
    w = np.random.default_rng(6).normal(0, 0.02, (N, K)).astype(np.float32)
    payload, scales = q4.gptq_pack(w, X, bits, group)
    P, S = torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda()
    deq = q4.qdequant(P, S, (N, K), bits, group)
    x = X[:5].copy()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.qgemm(torch.from_numpy(x).cuda(), P, S, N, K, bits, group, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rd = oracle.dequant(payload, scales, N * K, bits, group).reshape(N, K)
    assert np.array_equal(deq.cpu().numpy().view(np.uint32), rd.view(np.uint32))
    yref, bound = oracle.qgemm(x, payload, scales, N, K, bits, group)
    assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - yref) <= 1e-5 * bound + 1e-6)
