"""The whole-stack decode driver: one CUDA graph per token step replays the same qgemm
calls as an eager step, and a matrix of the stack (packed on the GPU) matches the oracle."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def test_graph_step_runs_and_matches_oracle_on_one_matrix():
    import torch

    import int4_quantized_b200 as q4
    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(4, 128, layers=1)
    assert len(stack) == 7 and [(n, k) for n, k, _, _, _ in stack] == [(n, k) for _, n, k in ds.SHAPES]
    r = ds.time_stack(stack, 4, M=1, reps=2, warmup=1)
    assert r["gemvs"] == 7 and r["us_per_step"] > 0 and r["weight_bytes"] == ds.stack_bytes(stack)
    # the down projection (K = 11008) of layer 0 against the oracle
    N, K, g, payload, scales = stack[6]
    x = np.random.default_rng(1).normal(0, 1, (2, K)).astype(np.float32)
    y = q4.qgemm(torch.from_numpy(x).cuda(), payload, scales, N, K, 4, g)
    torch.cuda.synchronize()
    rows = list(range(0, N, 37))
    yref, bound = oracle.qgemm(x, payload.cpu().numpy(), scales.cpu().numpy(), N, K, 4, g, rows=rows)
    err = np.abs(y.cpu().numpy()[:, rows].astype(np.float64) - yref)
    assert np.all(err <= 1e-5 * bound + 1e-6)


def test_stack_bytes_of_the_full_stack_shapes():
    from int4_quantized_b200 import decode_stack as ds

    n = sum(N * K for _, N, K in ds.SHAPES) * 32
    assert n == 6_476_005_376  # the Llama-7B-shaped stack's weights
