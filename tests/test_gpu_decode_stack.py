"""The whole-stack decode driver (int4_quantized_b200/decode_stack.py): the token step
replayed from a CUDA graph of qgemm calls, and the same step as one launch of the
decode-stack kernel, both checked GEMV by GEMV against the oracle on the x each GEMV read
(data flow: every layer reads what the layer before wrote), per element
|y - y_oracle| <= 1e-5 * sum_k |w'x| + 1e-6 on sampled rows."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-6


def check_step(stack, acts, bits, rows_per=48, seed=0):
    rng = np.random.default_rng(seed)
    for f in stack:
        x = acts.x_of(f).float().cpu().numpy().reshape(1, f.K)
        y = acts.y_of(f).cpu().numpy()
        assert np.all(np.isfinite(y)), f"L{f.layer}.{f.name}"
        rows = sorted(set(rng.choice(f.N, rows_per, replace=False).tolist()) | {0, f.N - 1})
        yref, bound = oracle.qgemm(x, f.payload.cpu().numpy(), f.scales.cpu().numpy(), f.N, f.K, bits, f.group,
                                   rows=rows)
        err = np.abs(y[rows].astype(np.float64).reshape(1, -1) - yref)
        lim = RTOL * bound + ATOL
        assert np.all(err <= lim), f"L{f.layer}.{f.name}: worst ratio {float((err / lim).max()):.3g}"


@pytest.mark.parametrize("bits,group", [(4, 128), (8, None)])
def test_graph_replayed_step_matches_oracle(bits, group):
    import torch

    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(bits, group, layers=2, sigma=1.0 / 64)
    acts = ds.Activations(stack)
    graph, stream, ncalls, keep = ds.capture_step(stack, bits, acts)
    assert ncalls == 8
    for y in acts.y.values():
        y.fill_(float("nan"))
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    check_step(stack, acts, bits)
    del graph, keep


@pytest.mark.parametrize("fused", [False, True])
def test_persistent_step_matches_oracle(fused):
    import torch

    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(4, 128, layers=2, sigma=1.0 / 64)
    dstack, acts = ds.make_decode_stack(stack, 4, fused=fused)
    assert len(dstack.gemvs) == (8 if fused else 14)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        dstack.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_step(stack, acts, 4)


def test_fused_layout_is_the_separate_packing():
    # q|k|v packed into one buffer is byte for byte the three separate payloads
    import torch

    import int4_quantized_b200 as q4
    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(4, 128, layers=1)
    f = stack[0]
    assert f.name == "qkv" and f.N == 3 * 4096
    for i, m in enumerate(f.parts):
        gen = torch.Generator(device="cuda").manual_seed(100 + i)
        w = torch.randn(m.N, m.K, device="cuda", generator=gen) * 0.02
        p, s = q4.qpack(w, 4, 128)
        assert torch.equal(p, m.payload) and torch.equal(s.view(torch.int32), m.scales.view(torch.int32))


def test_stack_bytes_of_the_full_stack_shapes():
    from int4_quantized_b200 import decode_stack as ds

    n = sum(N * K for _, N, K in ds.SHAPES) * 32
    assert n == 6_476_005_376  # the Llama-7B-shaped stack's weights
