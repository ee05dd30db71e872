"""The prefill path of qgemm (bf16 x, M >= 64, K and group multiples of 64: the
tensor-memory GEMM) against the oracle's fp64 product with the dequantized weights.

Tolerance per output element: |y - y_oracle| <= 1e-5 * sum_k |w'[n,k] x[m,k]| + 1e-6
(the QuantizedMatmul of "Huit bits, puis quatre": the same numbers as the product with
the dequantized weights, up to the order of the sums). The oracle sees exactly the bf16
values the GPU receives.
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-6


@pytest.fixture(scope="module")
def q4():
    import int4_quantized_b200 as m

    m.lib()
    return m


def run_bf16(q4, x_bf16, payload, scales, N, K, bits, group):
    import torch

    xt = x_bf16.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.qgemm(xt, torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda(), N, K, bits, group,
                 status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"status word {int(status.item()):#x}: a bounded wait gave up"
    return y.cpu().numpy()


def check(q4, w, x_bf16, bits, group, rows=None, what=""):
    N, K = w.shape
    assert q4.qgemm_workspace_bytes(x_bf16.shape[0], N, K, bits, group, x_bf16.dtype) == 0  # the GEMM path
    payload, scales, _ = oracle.pack(w, bits, group)
    y = run_bf16(q4, x_bf16, payload, scales, N, K, bits, group)
    assert y.shape == (x_bf16.shape[0], N) and np.all(np.isfinite(y))
    xin = x_bf16.float().numpy()
    yref, bound = oracle.qgemm(xin, payload, scales, N, K, bits, group, rows=rows)
    ysel = y if rows is None else y[:, rows]
    err = np.abs(ysel.astype(np.float64) - yref)
    lim = RTOL * bound + ATOL
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{what}: {len(bad)} outside tolerance, worst {float((err / lim).max()):.3g} at {bad[:4].tolist()}"


def bf16(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 128), (4, 64), (8, 1024), (8, 64), (4, 1024)])
def test_ragged_shapes(q4, bits, group):
    # M and N not multiples of the 256 x 128 output tile
    rng = np.random.default_rng(bits * 7 + group)
    for M, N in ((300, 200), (64, 130), (257, 1)):
        w = rng.normal(0, 0.02, (N, 1024)).astype(np.float32)
        w.reshape(-1)[rng.choice(w.size, max(1, w.size // 500), replace=False)] *= 20
        x = bf16(rng.normal(0, 1, (M, 1024)))
        check(q4, w, x, bits, group, what=f"M{M} N{N} int{bits} g{group}")


@pytest.mark.parametrize("bits,group", [(4, 128), (8, 256)])
def test_last_round_split_into_narrow_items(q4, bits, group):
    # 75 x 2 = 150 output tiles on a 148-SM grid: the 2 tiles of the last round are cut
    # into 4 narrower items each (64 activation rows); all of y is checked on sampled rows
    rng = np.random.default_rng(21 + bits)
    N, K, M = 128 * 75, 256, 512
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = bf16(rng.normal(0, 1, (M, K)))
    rows = sorted(set(range(0, 128)) | set(range(N - 256, N)) | set(rng.choice(N, 200, replace=False).tolist()))
    check(q4, w, x, bits, group, rows=rows, what=f"split int{bits} g{group}")


def test_one_hot_rows_select_dequantized_weights_exactly(q4):
    # x = e_k (exact in bf16): the MMA sum is the single code, times the group scale once,
    # so y[:, n] is w'[n, k] bit for bit -- any mix-up of k inside a tile shows here
    rng = np.random.default_rng(3)
    N, K = 256, 512
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    ks = [0, 1, 7, 8, 63, 64, 127, 200, 511] + list(range(300, 364))
    x = np.zeros((len(ks), K), np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    for bits, g in ((4, 128), (8, 512), (8, 64)):
        payload, scales, _ = oracle.pack(w, bits, g)
        y = run_bf16(q4, bf16(x), payload, scales, N, K, bits, g)
        wd = oracle.dequant_rows(payload, scales, N, K, bits, g)
        for i, k in enumerate(ks):
            assert np.array_equal(y[i].view(np.uint32), wd[:, k].view(np.uint32)), (bits, g, k)


def test_prefill_config_sampled(q4):
    # M = 2048, K = 4096, N = 14336, bf16 x; every row of y against sampled output channels
    wl = workloads.WORKLOADS["prefill"]
    m = wl.matrices[0]
    w = workloads.weight(m)
    x = workloads.activations_bf16(2048, m.K, wl.x_seed(m.K))
    rng = np.random.default_rng(11)
    rows = sorted(set(range(16)) | set(range(m.N - 16, m.N)) | set(rng.choice(m.N, 96, replace=False).tolist()))
    for bits, g in wl.formats:
        check(q4, w, x, bits, m.K if g is None else g, rows=rows, what=f"prefill int{bits}")


def test_large_activations_and_mixed_magnitudes(q4):
    rng = np.random.default_rng(9)
    w = rng.normal(0, 0.02, (192, 768)).astype(np.float32)
    for scale in (1e-20, 1e-3, 1e4, 1e20):
        x = bf16(rng.normal(0, 1, (96, 768)) * scale)
        check(q4, w, x, 4, 128, what=f"x scale {scale}")
    x = rng.normal(0, 1, (80, 768)).astype(np.float32)
    x[:, :300] *= 1e-12
    x[5, 17] = 6.0e4
    check(q4, w, bf16(x), 8, 768, what="mixed magnitudes")


def test_deterministic(q4):
    import torch

    rng = np.random.default_rng(4)
    N, K, M = 640, 2048, 512
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    payload, scales, _ = oracle.pack(w, 4, 128)
    x = bf16(rng.normal(0, 1, (M, K))).cuda()
    P, S = torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda()
    y0 = q4.qgemm(x, P, S, N, K, 4, 128)
    y1 = q4.qgemm(x, P, S, N, K, 4, 128)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))
