"""qgemm with activations whose magnitudes differ by many orders inside one block of k.

The tolerance of every qgemm test is per output element,
|y_gpu - y_oracle| <= 1e-5 * sum_k |w'[n,k] x[m,k]| + 1e-6, so an activation that meets a
zero code contributes nothing to the bound. A matmul that rounds the activations relative
to the largest |x| of a block of k (fixed point) fails here: the huge activation sits on a
column whose code is 0 in most rows, so its size sets the rounding step of its neighbours
while the bound stays small. "Huit bits, puis quatre", section "Des valeurs aberrantes, à 29
millions de paramètres ?", describes exactly this failure for a rounded activation vector:
one large component rounded together with the rest ruins the precision of the whole
vector. The GPU path must keep every product's relative accuracy instead.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-6


@pytest.fixture(scope="module")
def q4():
    import int4_quantized_b200 as m

    m.lib()
    return m


def run(q4, x, payload, scales, N, K, bits, group, bf16=False, static=False):
    import torch

    xt = torch.from_numpy(x).cuda()
    if bf16:
        xt = xt.to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.qgemm(xt, torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda(), N, K, bits, group,
                 status=status, weights_static=static)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y.cpu().numpy()


def check(q4, w, x, bits, group, what):
    N, K = w.shape
    payload, scales, _ = oracle.pack(w, bits, group)
    y = run(q4, x, payload, scales, N, K, bits, group)
    yref, bound = oracle.qgemm(x, payload, scales, N, K, bits, group)
    err = np.abs(y.astype(np.float64) - yref)
    lim = RTOL * bound + ATOL
    bad = np.argwhere(err > lim)
    assert bad.size == 0, (f"{what}: {len(bad)} of {err.size} outside tolerance, worst ratio "
                           f"{float((err / lim).max()):.3g} at {bad[:3].tolist()}")


def weights_with_zero_columns(N, K, cols, seed, zero_frac=0.9):
    """W ~ N(0, 0.02) whose columns `cols` are 0 in `zero_frac` of the rows (code 0 there)."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    for c in cols:
        w[rng.random(N) < zero_frac, c] = 0.0
    return w


@pytest.mark.parametrize("K", [1024, 4096])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8])
@pytest.mark.parametrize("ratio", [1e6, 1e7])
def test_huge_activation_on_zero_code_column(q4, K, bits, M, ratio):
    # one activation per 1024 k is `ratio` times its neighbours and meets a code of 0 in
    # 90 % of the rows
    N = 384
    cols = [137 + 1024 * b for b in range(K // 1024)]
    w = weights_with_zero_columns(N, K, cols, seed=K + bits + M)
    rng = np.random.default_rng(K * 7 + M)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    for c in cols:
        x[:, c] = ratio * (1.0 + rng.random(M)).astype(np.float32)
    check(q4, w, x, bits, 128, f"K{K} int{bits} g128 M{M} ratio {ratio:g}")


@pytest.mark.parametrize("bits,group", [(4, 128), (8, 128), (8, 1024)])
@pytest.mark.parametrize("M", [1, 3])
def test_small_activations_with_one_large(q4, bits, group, M):
    # x ~ N(0, 1e-3) with one 1e4 entry where most rows have a zero code: the bound is a
    # few 1e-6 while the large entry is 1e7 times the rest
    N, K = 256, 1024
    w = weights_with_zero_columns(N, K, [500], seed=bits * 31 + M, zero_frac=0.95)
    rng = np.random.default_rng(group + M)
    x = rng.normal(0, 1e-3, (M, K)).astype(np.float32)
    x[:, 500] = 1e4
    check(q4, w, x, bits, group, f"int{bits} g{group} M{M}")


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 8])
def test_block_range_of_two_to_the_thirty(q4, bits, M):
    # in every row of x the largest |x| of each block of 1024 k is 2^30 times its
    # smallest nonzero entries; the largest sits on a zero-code column, and half the
    # block holds the smallest values
    N, K = 320, 2048
    cols = [3, 1024 + 900]
    w = weights_with_zero_columns(N, K, cols, seed=bits + 10 * M, zero_frac=1.0)
    rng = np.random.default_rng(bits * 3 + M)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    x[:, ::2] = np.float32(2.0 ** -30) * np.sign(x[:, ::2] + 1e-30)
    for c in cols:
        x[:, c] = 1.0
    check(q4, w, x, bits, 128, f"2^30 range int{bits} M{M}")


@pytest.mark.parametrize("M", [1, 4])
def test_magnitudes_across_the_fp32_range(q4, M):
    # every k gets its own magnitude, from 1e-30 to 1e30, in a random order
    N, K = 256, 2048
    rng = np.random.default_rng(40 + M)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    mag = 10.0 ** rng.uniform(-30, 30, (M, K))
    x = (rng.normal(0, 1, (M, K)) * mag).astype(np.float32)
    for bits, g in ((4, 128), (8, 2048), (4, 32)):
        check(q4, w, x, bits, g, f"fp32 range int{bits} g{g} M{M}")


def test_subnormal_activations(q4):
    # activations down to the fp32 subnormal range add at most 2^-126-sized errors
    N, K = 128, 1024
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = (rng.normal(0, 1, (2, K)) * 1e-40).astype(np.float32)
    x[1, :8] = 1.0
    check(q4, w, x, 4, 128, "subnormal x")
