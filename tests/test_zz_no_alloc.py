"""qgemm_noalloc (built-in device scratch, no allocation in the call) against qgemm.

Both entry points run the same kernels on the same plan, so their results must agree bit
for bit; here the no-allocation one is called through the C ABI twice in a row, on
different problems so that the second call finds what the first left in the shared
scratch, and each result is compared with qgemm's bit for bit. The file name sorts last
so the scratch is also exercised after the rest of the suite has run.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-6


@pytest.fixture(scope="module")
def q4():
    import int4_quantized_b200 as m

    m.lib()
    return m


def problem(q4, M, N, K, bits, group, bf16, seed):
    import torch

    g = torch.Generator(device="cpu").manual_seed(seed)
    w = (torch.randn(N, K, generator=g) * 0.02).cuda()
    x = torch.randn(M, K, generator=g).cuda()
    if bf16:
        x = x.to(torch.bfloat16)
    payload, scales = q4.qpack(w, bits, group)
    wq = q4.qdequant(payload, scales, (N, K), bits, group)
    bound = (wq.double().abs() @ x.double().abs().T).T.cpu().numpy()
    return x, payload, scales, bound


def call_noalloc_abi(q4, x, payload, scales, N, K, bits, group, y):
    import torch

    xt = q4.Q4_X_BF16 if x.dtype == torch.bfloat16 else q4.Q4_X_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return q4.lib().qgemm_noalloc(ctypes.c_void_p(x.data_ptr()), xt, x.shape[0],
                                  ctypes.c_void_p(payload.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                  N, K, bits, group, ctypes.c_void_p(y.data_ptr()), None, stream)


CASES = [
    # M, N, K, bits, group, bf16
    (1, 4096, 4096, 4, 128, False),
    (8, 1000, 2048, 8, 128, False),
    (16, 304, 4096, 4, 32, True),
    (3, 11008, 4096, 8, 4096, False),
    (1, 256, 2048, 4, 4096, False),   # groups of two whole rows: expanded row scales at the start
    (96, 256, 1024, 4, 128, True),    # bf16 x, M >= 64: the tensor-core GEMM (no scratch used)
]


@pytest.mark.parametrize("first,second", [(0, 1), (2, 3), (1, 0), (1, 4), (4, 2), (5, 4)])
def test_noalloc_matches_qgemm_two_calls(q4, first, second):
    import torch

    probs = []
    for i, idx in enumerate((first, second)):
        M, N, K, bits, group, bf16 = CASES[idx]
        probs.append((CASES[idx], problem(q4, M, N, K, bits, group, bf16, seed=100 + 10 * idx + i)))
    outs = []
    for (M, N, K, bits, group, _), (x, payload, scales, _) in probs:
        y = torch.full((M, N), float("nan"), device="cuda")
        st = call_noalloc_abi(q4, x, payload, scales, N, K, bits, group, y)
        assert st == q4.Q4_OK, q4.lib().q4_status_str(st).decode()
        outs.append(y)
    torch.cuda.synchronize()
    for ((M, N, K, bits, group, _), (x, payload, scales, bound)), y in zip(probs, outs):
        yref = q4.qgemm(x, payload, scales, N, K, bits, group)
        torch.cuda.synchronize()
        a, b = y.cpu().numpy(), yref.cpu().numpy()
        assert np.isfinite(a).all()
        # the same kernels on the same inputs: the same bits, whatever the last call left
        # in the shared scratch
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"M={M} N={N} K={K} bits={bits} g={group}"
        a64 = a.astype(np.float64)
        assert np.all(np.abs(a64 - b.astype(np.float64)) <= RTOL * bound + ATOL)


def test_noalloc_allocates_nothing(q4):
    import torch

    M, N, K, bits, group, bf16 = CASES[0]
    x, payload, scales, _ = problem(q4, M, N, K, bits, group, bf16, seed=7)
    y = torch.empty(M, N, device="cuda")
    assert call_noalloc_abi(q4, x, payload, scales, N, K, bits, group, y) == q4.Q4_OK
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert call_noalloc_abi(q4, x, payload, scales, N, K, bits, group, y) == q4.Q4_OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0


def test_noalloc_rejects_beyond_scratch(q4):
    import torch

    M, N, K, bits, group = 64, 128, 16384, 4, 128
    need = q4.qgemm_workspace_bytes(M, N, K, bits, group)
    assert need > q4.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(M, K, device="cuda")
    payload = torch.zeros(N * K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.ones(N * K // group, device="cuda")
    y = torch.full((M, N), 5.0, device="cuda")
    st = call_noalloc_abi(q4, x, payload, scales, N, K, bits, group, y)
    assert st == q4.Q4_ERR_SCRATCH_LIMIT
    assert "scratch" in q4.lib().q4_status_str(st).decode()
    torch.cuda.synchronize()
    assert bool((y == 5.0).all())  # nothing was enqueued
