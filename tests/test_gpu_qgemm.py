"""qgemm on the GPU vs the oracle's fp64 matmul with the dequantized weights (the
QuantizedMatmul of "Huit bits, puis quatre": same numbers up to summation order).

Tolerance, per output element: |y_gpu - y_oracle| <= 1e-5 * sum_k |w'[n,k] x[m,k]| + 1e-6.
The packed weights fed to the GPU come from the oracle, so this isolates the matmul.
Full-size problems are checked on sampled output channels, computed one by one by the
oracle.
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


def run_gpu(q4, x, payload, scales, N, K, bits, group, bf16=False):
    import torch

    xt = torch.from_numpy(x).cuda()
    if bf16:
        xt = xt.to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.qgemm(xt, torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda(), N, K, bits, group,
                 status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"status word {int(status.item()):#x}: a bounded wait gave up"
    return y.cpu().numpy()


def check(y, yref, bound, what):
    err = np.abs(y.astype(np.float64) - yref)
    lim = RTOL * bound + ATOL
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{what}: {len(bad)} outside tolerance, worst ratio {float((err / lim).max()):.3g} at {bad[:3].tolist()}"
    return float((err / lim).max())


def sample_rows(N, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(range(min(16, N))) | set(range(max(0, N - 16), N))
    rows |= set(rng.choice(N, min(k, N), replace=False).tolist())
    return sorted(rows)


def case(q4, w, x, bits, group, rows=None, bf16=False, what=""):
    N, K = w.shape
    payload, scales, _ = oracle.pack(w, bits, group)
    xin = x
    if bf16:
        import torch

        xin = torch.from_numpy(x).to(torch.bfloat16).float().numpy()  # the values the GPU sees
    y = run_gpu(q4, x, payload, scales, N, K, bits, group, bf16=bf16)
    assert y.shape == (x.shape[0], N)
    yref, bound = oracle.qgemm(xin, payload, scales, N, K, bits, group, rows=rows)
    ysel = y if rows is None else y[:, rows]
    assert np.all(np.isfinite(y))
    return check(ysel, yref, bound, what)


def test_small_config_full(q4):
    wl = workloads.WORKLOADS["small"]
    w = workloads.weight(wl.matrices[0])
    x = workloads.activations(1, 1024, wl.x_seed(1024))
    for bits, g in wl.formats:
        case(q4, w, x, bits, g, what=f"small int{bits} g{g}")


@pytest.mark.parametrize("M", [1, 8])
def test_mid_config_full(q4, M):
    wl = workloads.WORKLOADS["mid"]
    w = workloads.weight(wl.matrices[0])
    x = workloads.activations(M, 4096, wl.x_seed(4096))
    for bits, g in wl.formats:
        case(q4, w, x, bits, g, what=f"mid int{bits} g{g} M{M}")


@pytest.mark.parametrize("idx", [0, 4, 6])   # q (4096x4096), gate (11008x4096), down (4096x11008)
# M = 4, 8, 10: one to four column blocks, one CTA per SM on 4096 rows and two on 11008
@pytest.mark.parametrize("M", [1, 4, 8, 10, 16])
def test_llama7b_sampled(q4, idx, M):
    wl = workloads.WORKLOADS["llama7b"]
    m = wl.matrices[idx]
    w = workloads.weight(m)
    x = workloads.activations(M, m.K, wl.x_seed(m.K))
    rows = sample_rows(m.N, 200, idx)
    for bits, g in wl.formats:
        case(q4, w, x, bits, m.K if g is None else g, rows=rows, what=f"{m.name} int{bits} M{M}")


@pytest.mark.parametrize("which", [0, 2])
def test_mlp70b_sampled(q4, which):
    wl = workloads.WORKLOADS["mlp70b"]
    m = wl.matrices[which]
    w = workloads.weight(m)
    x = workloads.activations(1, m.K, wl.x_seed(m.K))
    case(q4, w, x, 4, 64, rows=sample_rows(m.N, 300, which), what=m.name)


@pytest.mark.parametrize("M", [1, 9, 40, 300])
def test_row_counts(q4, M):
    # the codes path is checked for 1, 9, 40 and 300 activation rows ("Huit bits, puis
    # quatre", section "Ranger des entiers dans des f32")
    rng = np.random.default_rng(M)
    w = rng.normal(0, 0.02, (512, 1024)).astype(np.float32)
    x = rng.normal(0, 1, (M, 1024)).astype(np.float32)
    for bits, g in ((4, 128), (8, 1024), (4, 32), (8, 64)):
        case(q4, w, x, bits, g, what=f"M{M} int{bits} g{g}")


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (4, 128), (4, 256), (4, 4096),
                                        (8, 32), (8, 64), (8, 96), (8, 128), (8, 4096), (4, 96), (4, 384)])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 16])
def test_group_variants(q4, bits, group, M):
    rng = np.random.default_rng(bits * 1000 + group + M)
    N, K = 200, (4608 if group % 96 == 0 else 4096)  # ragged N: not a multiple of 16
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w.reshape(-1)[rng.choice(N * K, 50, replace=False)] *= 20  # outliers
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    case(q4, w, x, bits, group, what=f"int{bits} g{group} M{M}")


@pytest.mark.parametrize("bits,group,K", [(4, 64, 4160), (4, 32, 4128), (8, 32, 4128), (8, 96, 4128 + 96 * 3)])
@pytest.mark.parametrize("M", [1, 3, 9])
def test_partial_last_stage(q4, bits, group, K, M):
    # rows whose byte length is not a multiple of the 128-byte stage: the last stage of
    # every row is partly outside the payload
    if K % group:
        K = group * (K // group)
    rng = np.random.default_rng(K + bits + M)
    w = rng.normal(0, 0.02, (136, K)).astype(np.float32)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    case(q4, w, x, bits, group, what=f"K{K} int{bits} g{group} M{M}")


@pytest.mark.parametrize("bits,group", [(4, 32), (8, 32), (4, 64), (4, 128)])
@pytest.mark.parametrize("M", [2, 9])
def test_many_k_blocks_per_cta(q4, bits, group, M):
    # 152 x 128 output rows fill the grid without a K split: each CTA streams all of K
    # through its rings, crossing many k-blocks (scale buffers reused several times)
    # before and after its ring of codes and digits wraps
    N, K = 152 * 128, 2048
    rng = np.random.default_rng(bits * 100 + group + M)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    case(q4, w, x, bits, group, rows=sample_rows(N, 200, M), what=f"int{bits} g{group} M{M}")


@pytest.mark.parametrize("M", [1, 16, 40, 64, 128])
def test_bf16_activations(q4, M):
    rng = np.random.default_rng(77 + M)
    w = rng.normal(0, 0.02, (384, 2048)).astype(np.float32)
    x = rng.normal(0, 1, (M, 2048)).astype(np.float32)
    for bits, g in ((4, 128), (8, 2048)):
        case(q4, w, x, bits, g, bf16=True, what=f"bf16 M{M} int{bits}")


def test_activation_range_extremes(q4):
    # tiny, huge and mixed-magnitude activations: each activation is split exactly into
    # three bf16 pieces, so every product keeps its own exponent
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, (64, 512)).astype(np.float32)
    for scale in (1e-30, 1e-8, 1e-3, 1e4, 1e30):
        x = (rng.normal(0, 1, (3, 512)) * scale).astype(np.float32)
        case(q4, w, x, 4, 128, what=f"x scale {scale}")
    x = rng.normal(0, 1, (2, 512)).astype(np.float32)
    x[0, :256] *= 1e-12
    x[1, 7] = 6.0e4
    case(q4, w, x, 8, 64, what="mixed magnitudes")
    x = np.zeros((2, 512), np.float32)
    case(q4, w, x, 4, 128, what="zeros")


def test_one_hot_selects_dequantized_weight_exactly(q4):
    # with x = e_k the only product is code * 1, scaled once by the fp32 scale:
    # y[:, n] equals w'[n, k] bit for bit
    wl = workloads.WORKLOADS["mid"]
    w = workloads.weight(wl.matrices[0])
    for bits, g in wl.formats:
        payload, scales, _ = oracle.pack(w, bits, g)
        for k in (0, 1, 127, 4095):
            x = np.zeros((1, 4096), np.float32)
            x[0, k] = 1.0
            y = run_gpu(q4, x, payload, scales, 4096, 4096, bits, g)
            col = oracle.dequant_rows(payload, scales, 4096, 4096, bits, g)[:, k]
            assert np.array_equal(y[0].view(np.uint32), col.view(np.uint32)), (bits, k)


def test_empty_shapes(q4):
    import torch

    p = torch.zeros(64 * 64, dtype=torch.uint8, device="cuda")
    s = torch.ones(64 * 64 // 32, dtype=torch.float32, device="cuda")
    y = q4.qgemm(torch.zeros((0, 128), device="cuda"), p, s, 64, 128, 4, 32)
    assert y.shape == (0, 64)


def test_deterministic(q4):
    rng = np.random.default_rng(9)
    w = rng.normal(0, 0.02, (4096, 4096)).astype(np.float32)
    x = rng.normal(0, 1, (8, 4096)).astype(np.float32)
    payload, scales, _ = oracle.pack(w, 4, 128)
    a = run_gpu(q4, x, payload, scales, 4096, 4096, 4, 128)
    b = run_gpu(q4, x, payload, scales, 4096, 4096, 4, 128)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rows_per_group", ["all", 2, 8])
@pytest.mark.parametrize("M,bf16", [(1, False), (5, False), (96, True)])
def test_groups_of_whole_rows(q4, bits, rows_per_group, M, bf16):
    # one scale for the whole matrix (the INT4_TENSOR format) or one per few rows
    import torch

    N, K = 320, 512
    g = N * K if rows_per_group == "all" else rows_per_group * K
    rng = np.random.default_rng(M * 10 + bits)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    w.reshape(-1)[rng.choice(N * K, 40, replace=False)] *= 20
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    payload, scales, _ = oracle.pack(w, bits, g)
    assert scales.size == N * K // g
    xin = torch.from_numpy(x).to(torch.bfloat16).float().numpy() if bf16 else x
    xt = torch.from_numpy(x).cuda()
    if bf16:
        xt = xt.to(torch.bfloat16)
    P, S = torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = q4.qgemm(xt, P, S, N, K, bits, g, status=status)
    y2 = q4.qgemm(xt, P, S, N, K, bits, g, status=status, weights_static=True)
    y3 = torch.empty_like(y)
    q4.qgemm_noalloc(xt, P, S, N, K, bits, g, y3, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yref, bound = oracle.qgemm(xin, payload, scales, N, K, bits, g)
    check(y.cpu().numpy(), yref, bound, f"int{bits} g{g} M{M}")
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    assert torch.equal(y.view(torch.int32), y3.view(torch.int32))


ANY_GROUP = [
    # M, N, K, bits, group, bf16 x -- groups the fused paths do not take
    (1, 64, 256, 4, 16, False),       # narrower than a 32-wide segment
    (3, 96, 256, 8, 48, False),       # 48 does not divide K: groups cross rows at varying offsets
    (5, 66, 256, 4, 384, False),      # 3K/2: every other row starts mid-group
    (2, 30, 77, 4, 10, False),        # odd K: int4 rows start in the middle of a byte
    (1, 7, 3, 8, 7, False),           # groups longer than a row, tiny
    (17, 33, 100, 4, 50, True),       # K % 32 != 0, bf16 x
    (70, 64, 96, 4, 1, True),         # one scale per weight, many rows of x
    (9, 12, 100, 8, 100, False),      # per-row scales with K % 32 != 0
    (1, 257, 1000, 4, 40, False),     # groups of 40 crossing rows, ragged sizes
    (8, 2048, 2048, 4, 16, False),    # a larger one (scales of 16 weights)
]


@pytest.mark.parametrize("idx", range(len(ANY_GROUP)))
def test_any_group(q4, idx):
    # every group that qpack accepts, through the any-group kernel, against the oracle's
    # dequantization of the flattened tensor (groups cut across rows as pack() cuts them)
    M, N, K, bits, g, bf16 = ANY_GROUP[idx]
    rng = np.random.default_rng(700 + idx)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    payload, scales, _ = oracle.pack(w, bits, g)
    xin = x
    if bf16:
        import torch

        xin = torch.from_numpy(x).to(torch.bfloat16).float().numpy()  # the values the GPU reads
    y = run_gpu(q4, x, payload, scales, N, K, bits, g, bf16=bf16)
    yref, bound = oracle.qgemm(xin, payload, scales, N, K, bits, g)
    check(y, yref, bound, f"any group M={M} N={N} K={K} int{bits} g={g}")
    assert q4.qgemm_workspace_bytes(M, N, K, bits, g) == 0
