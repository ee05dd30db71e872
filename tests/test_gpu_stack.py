"""The decode stack (q4_stack_prepare / q4_stack_run): every GEMV of a decode step in one
persistent kernel, against the oracle's fp64 matmul ("Huit bits, puis quatre", sections
"Ranger des entiers dans des f32" and "La vitesse").

The stacks here have data flow: each level reads what the level before it wrote (a
transformer layer's q|k|v, o, gate|up, down, with the attention and the activation
function replaced by reading one of the previous outputs). Every GEMV is checked against
the oracle given exactly the x the GPU read, per output element:
|y_gpu - y_oracle| <= 1e-5 * sum_k |w'[n,k] x[k]| + 1e-6.
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


def layer_shapes(d, f):
    # (name, N, K, level offset, x source) -- x source: "h" (the layer input), or the name
    # of an earlier GEMV's output
    return [("q", d, d, 0, "h"), ("k", d, d, 0, "h"), ("v", d, d, 0, "h"), ("o", d, d, 1, "q"),
            ("gate", f, d, 2, "o"), ("up", f, d, 2, "o"), ("down", d, f, 3, "gate")]


def build(q4, layers, d, f, bits, group_of, seed, x_dtype=None):
    """Seeded weights packed by the oracle, the stack's buffers and its GEMV list.

    W ~ N(0, 1/K), so that the activations keep their size through the layers."""
    import torch

    x_dtype = x_dtype or torch.float32
    rng = np.random.default_rng(seed)
    h = torch.from_numpy(rng.normal(0, 1, d).astype(np.float32)).cuda().to(x_dtype)
    # bf16 stacks read bf16 activations, which an fp32 output cannot provide: every GEMV
    # then reads a fixed bf16 input of its K
    hk = {K: torch.from_numpy(rng.normal(0, 1, K).astype(np.float32)).cuda().to(x_dtype) for K in (d, f)}
    gemvs, host = [], []
    prev = {"h": h}
    for layer in range(layers):
        outs = {}
        for name, N, K, lo, src in layer_shapes(d, f):
            w = rng.normal(0, 1.0 / np.sqrt(K), (N, K)).astype(np.float32)
            g = group_of(K)
            p, s, _ = oracle.pack(w, bits, g)
            P, S = torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda()
            x = prev[src] if src == "h" else outs[src]
            if x_dtype != torch.float32:
                x = hk[K]
            y = torch.empty(N, dtype=torch.float32, device="cuda")
            outs[name] = y
            gemvs.append(q4.StackGemv(P, S, x, y, N, K, g, 4 * layer + lo))
            host.append((name, layer, N, K, g, p, s))
        prev = {"h": outs["down"] if x_dtype == torch.float32 else prev["h"]}
    return gemvs, host


def check_all(gemvs, host, bits, what):
    import torch

    worst = 0.0
    for gv, (name, layer, N, K, g, p, s) in zip(gemvs, host):
        x = gv.x.float().cpu().numpy().reshape(1, K)
        y = gv.y.cpu().numpy().reshape(1, N)
        assert np.all(np.isfinite(y)), f"{what} L{layer}.{name}: non-finite y"
        yref, bound = oracle.qgemm(x, p, s, N, K, bits, g)
        err = np.abs(y.astype(np.float64) - yref)
        lim = RTOL * bound + ATOL
        bad = np.argwhere(err > lim)
        assert bad.size == 0, (f"{what} L{layer}.{name}: {len(bad)} of {N} outside tolerance, worst ratio "
                               f"{float((err / lim).max()):.3g} at {bad[:3].tolist()}")
        worst = max(worst, float((err / lim).max()))
    return worst


CASES = [
    # bits, group rule, description
    (4, lambda K: 128, "int4 g128"),
    (8, lambda K: K, "int8 per channel"),
    (4, lambda K: 64, "int4 g64"),
    (4, lambda K: 32, "int4 g32"),
    (8, lambda K: 64, "int8 g64"),
    (8, lambda K: 32, "int8 g32"),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_small_stack_with_data_flow(q4, case):
    import torch

    bits, group_of, what = CASES[case]
    # d = 512, f = 1408: K = 1408 ends in a partial 128-byte tile at int4
    gemvs, host = build(q4, 3, 512, 1408, bits, group_of, seed=10 + case)
    st = q4.DecodeStack(gemvs, bits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_all(gemvs, host, bits, what)


def test_bf16_activations(q4):
    import torch

    gemvs, host = build(q4, 2, 512, 1408, 4, lambda K: 128, seed=3, x_dtype=torch.bfloat16)
    st = q4.DecodeStack(gemvs, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_all(gemvs, host, 4, "bf16 x")


def test_ragged_shapes_one_level(q4):
    # many GEMVs of odd row counts in a single level, and tiny levels with fewer tiles than
    # CTAs: row blocks split over CTAs at every offset
    import torch

    rng = np.random.default_rng(5)
    gemvs, host = [], []
    x = torch.from_numpy(rng.normal(0, 1, 1024).astype(np.float32)).cuda()
    level = 0
    for i, N in enumerate([1, 7, 129, 300, 1000, 77, 4096, 3]):
        w = rng.normal(0, 0.02, (N, 1024)).astype(np.float32)
        p, s, _ = oracle.pack(w, 4, 128)
        y = torch.empty(N, dtype=torch.float32, device="cuda")
        gemvs.append(q4.StackGemv(torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda(), x, y, N, 1024, 128, level))
        host.append((f"m{i}", 0, N, 1024, 128, p, s))
        if i in (2, 5):
            level += 1  # small levels (fewer tiles than CTAs) between larger ones
    st = q4.DecodeStack(gemvs, 4)
    st.run()
    torch.cuda.synchronize()
    check_all(gemvs, host, 4, "ragged")


def test_replays_are_bit_identical_and_graph_capturable(q4):
    import torch

    gemvs, host = build(q4, 2, 512, 1408, 4, lambda K: 128, seed=21)
    st = q4.DecodeStack(gemvs, 4)
    st.run()
    torch.cuda.synchronize()
    first = [g.y.clone() for g in gemvs]
    for _ in range(3):
        st.run()
    torch.cuda.synchronize()
    for a, g in zip(first, gemvs):
        assert torch.equal(a.view(torch.int32), g.y.view(torch.int32))
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        st.run()
    for g in gemvs:
        g.y.zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for a, g in zip(first, gemvs):
        assert torch.equal(a.view(torch.int32), g.y.view(torch.int32))
    check_all(gemvs, host, 4, "graph")


def test_wait_limit_gives_up_and_workspace_stays_usable(q4):
    # with a bound of 0 ns the level waits give up (the earlier level is still running):
    # the launch ends, Q4_STATUS_TIMEOUT is set, and the next run with the default bound
    # is exact again (the counters were returned to zero)
    import torch

    gemvs, host = build(q4, 2, 512, 1408, 4, lambda K: 128, seed=22)
    st = q4.DecodeStack(gemvs, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = [g.y.clone() for g in gemvs]
    st.set_wait_limit(0)
    st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) & q4.STATUS_TIMEOUT
    st.set_wait_limit(10 ** 9)
    status.zero_()
    for _ in range(2):
        st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for a, g in zip(ref, gemvs):
        assert torch.equal(a.view(torch.int32), g.y.view(torch.int32))


def test_llama7b_stack_sampled(q4):
    # the full Llama-7B-shaped step (32 layers x 7 GEMVs, int4 g128, 3.4 GB of packed
    # weights drawn on the device and packed by qpack); sampled rows of the first, a middle
    # and the last layer against the oracle on the x each GEMV read
    import torch

    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(4, 128, 32, torch.device("cuda"))
    dstack, acts = ds.make_decode_stack(stack, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dstack.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(0)
    for idx in (0, 3, 4, 6, 7 * 16 + 5, 7 * 31 + 6):
        g = dstack.gemvs[idx]
        N, K = g.N, g.K
        p = g.payload.cpu().numpy()
        s = g.scales.cpu().numpy()
        rows = sorted(set(rng.choice(N, 64, replace=False).tolist()) | {0, N - 1})
        x = g.x.float().cpu().numpy().reshape(1, K)
        yref, bound = oracle.qgemm(x, p, s, N, K, 4, 128, rows=rows)
        y = g.y.cpu().numpy()[rows].astype(np.float64).reshape(1, -1)
        err = np.abs(y - yref)
        assert np.all(err <= RTOL * bound + ATOL), f"GEMV {idx}: worst ratio {(err / (RTOL * bound + ATOL)).max():.3g}"


def test_llama7b_int8_per_channel_sampled(q4):
    # the full step at int8 with one scale per output channel (6.5 GB): the kernel variant
    # with five tiles in flight, whose CTAs build the slots of q|k|v and gate|up in several
    # chunks (more tiles per CTA than fit at once)
    import torch

    from int4_quantized_b200 import decode_stack as ds

    stack = ds.build_stack(8, None, 32, torch.device("cuda"))
    dstack, acts = ds.make_decode_stack(stack, 8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        dstack.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(1)
    for idx in (0, 2, 4, 6, 7 * 17 + 4, 7 * 31 + 6):
        g = dstack.gemvs[idx]
        N, K = g.N, g.K
        p = g.payload.cpu().numpy()
        s = g.scales.cpu().numpy()
        rows = sorted(set(rng.choice(N, 48, replace=False).tolist()) | {0, N - 1})
        x = g.x.float().cpu().numpy().reshape(1, K)
        yref, bound = oracle.qgemm(x, p, s, N, K, 8, K, rows=rows)
        y = g.y.cpu().numpy()[rows].astype(np.float64).reshape(1, -1)
        err = np.abs(y - yref)
        assert np.all(err <= RTOL * bound + ATOL), f"GEMV {idx}: worst ratio {(err / (RTOL * bound + ATOL)).max():.3g}"


def test_slots_built_in_chunks(q4):
    # a level of 28672 x 8192 int4 g128 gives each CTA about 26 tiles, more than the slots
    # that fit in shared memory at once: the CTA builds them chunk by chunk; the next level
    # reads the first 8192 outputs through their parts
    import torch

    rng = np.random.default_rng(41)
    N1, K1, N2 = 28672, 8192, 1024
    w1 = rng.normal(0, 1 / np.sqrt(K1), (N1, K1)).astype(np.float32)
    w2 = rng.normal(0, 1 / np.sqrt(K1), (N2, K1)).astype(np.float32)
    p1, s1, _ = oracle.pack(w1, 4, 128)
    p2, s2, _ = oracle.pack(w2, 4, 128)
    del w1, w2
    x = torch.from_numpy(rng.normal(0, 1, K1).astype(np.float32)).cuda()
    y1 = torch.empty(N1, device="cuda")
    y2 = torch.empty(N2, device="cuda")
    gemvs = [q4.StackGemv(torch.from_numpy(p1).cuda(), torch.from_numpy(s1).cuda(), x, y1, N1, K1, 128, 0),
             q4.StackGemv(torch.from_numpy(p2).cuda(), torch.from_numpy(s2).cuda(), y1[:K1], y2, N2, K1, 128, 1)]
    st = q4.DecodeStack(gemvs, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows1 = sorted(set(rng.choice(N1, 96, replace=False).tolist()) | {0, N1 - 1})
    for g, pk, sk, N, rows in ((gemvs[0], p1, s1, N1, rows1), (gemvs[1], p2, s2, N2, None)):
        xh = g.x.float().cpu().numpy().reshape(1, K1)
        yref, bound = oracle.qgemm(xh, pk, sk, N, K1, 4, 128, rows=rows)
        y = g.y.cpu().numpy()
        y = (y if rows is None else y[rows]).astype(np.float64).reshape(1, -1)
        err = np.abs(y - yref)
        assert np.all(err <= RTOL * bound + ATOL), f"worst ratio {(err / (RTOL * bound + ATOL)).max():.3g}"


@pytest.mark.parametrize("bits", [4, 8])
def test_stages_of_every_activation_range(q4, bits):
    # per 128-byte stage the kernel takes exact integer digits when the stage's activations
    # span at most 2^21, else exact bf16 pieces: stages of ordinary, zero, tiny, huge and
    # adversarial activations (one 1e7 on a column of zero codes) side by side, in a
    # two-level stack whose second level reads the first one's output
    import torch

    rng = np.random.default_rng(11 + bits)
    stagek = 256 if bits == 4 else 128
    K, N = 12 * stagek, 640
    x = rng.normal(0, 1, K).astype(np.float32)
    st = lambda i: slice(i * stagek, (i + 1) * stagek)
    x[st(1)] = 0.0                                      # all zero
    x[st(2)] *= np.float32(1e-30)                        # tiny
    x[st(3)] *= np.float32(1e30)                         # huge
    x[st(4)][::3] *= np.float32(2.0 ** -20)               # range just inside 2^21
    x[st(5)][::3] *= np.float32(2.0 ** -23)               # range just outside
    zero_col = 6 * stagek + 17
    x[zero_col] = 1e7                                   # huge activation on a zero-code column
    x[st(7)][::5] = 0.0                                  # exact zeros among normal values
    x[st(8)] = x[st(8)].astype(np.float32) * np.float32(3e-20)
    w = rng.normal(0, 1 / np.sqrt(K), (N, K)).astype(np.float32)
    w[:, zero_col] = 0.0
    w2 = rng.normal(0, 1 / np.sqrt(N), (N, N)).astype(np.float32)
    p, s, _ = oracle.pack(w, bits, 128)
    p2, s2, _ = oracle.pack(w2, bits, 128)
    xd = torch.from_numpy(x).cuda()
    y1 = torch.empty(N, device="cuda")
    y2 = torch.empty(N, device="cuda")
    gemvs = [q4.StackGemv(torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda(), xd, y1, N, K, 128, 0),
             q4.StackGemv(torch.from_numpy(p2).cuda(), torch.from_numpy(s2).cuda(), y1, y2, N, N, 128, 1)]
    stack = q4.DecodeStack(gemvs, bits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stack.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_all(gemvs, [("w", 0, N, K, 128, p, s), ("w2", 0, N, N, 128, p2, s2)], bits, f"ranges int{bits}")


def test_x_read_as_slices_of_earlier_outputs(q4):
    # every way a level can read earlier outputs: a slice of one previous-level y at a
    # 16-byte offset from its start (read through that GEMV's parts), a slice at another
    # offset and a slice across two GEMVs' y (both read from y once the sums are written),
    # and outputs of two levels back. The levels are small (fewer tiles than CTAs), so
    # every row block is split into parts.
    import torch

    rng = np.random.default_rng(31)
    h = torch.from_numpy(rng.normal(0, 1, 1024).astype(np.float32)).cuda()
    Y = torch.zeros(1701, dtype=torch.float32, device="cuda")  # y of A, one unused float, y of B
    yC = torch.empty(300, dtype=torch.float32, device="cuda")
    spec = [  # name, N, K, level, x
        ("A", 1000, 1024, 0, h), ("B", 700, 1024, 0, h),
        ("C", 300, 512, 1, Y[8:520]),        # A's rows 8..519: through A's parts
        ("D", 64, 256, 1, Y[1004:1260]),     # B's rows 3..258: B's y is not 16-byte aligned
        ("E", 130, 256, 1, Y[992:1248]),     # across A, the unused float and B
        ("F", 200, 512, 2, Y[0:512]),        # two levels back
        ("G", 96, 256, 2, yC[0:256]),        # C's rows 0..255: through C's parts
    ]
    outs = {"A": Y[:1000], "B": Y[1001:], "C": yC}
    gemvs, host = [], []
    for name, N, K, lvl, x in spec:
        assert x.data_ptr() % 16 == 0
        w = rng.normal(0, 1.0 / np.sqrt(K), (N, K)).astype(np.float32)
        p, s, _ = oracle.pack(w, 4, 128)
        y = outs.get(name)
        if y is None:
            y = torch.empty(N, dtype=torch.float32, device="cuda")
        gemvs.append(q4.StackGemv(torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda(), x, y, N, K, 128, lvl))
        host.append((name, lvl, N, K, 128, p, s))
    # an x that does not start on a 16-byte boundary is rejected up front
    bad = list(gemvs)
    bad[3] = q4.StackGemv(bad[3].payload, bad[3].scales, Y[1005:1261], bad[3].y, 64, 256, 128, 1)
    with pytest.raises(q4.Q4Error):
        q4.DecodeStack(bad, 4)
    st = q4.DecodeStack(gemvs, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert float(Y[1000]) == 0.0  # nobody writes between the two outputs
    check_all(gemvs, host, 4, "slices")


def test_y_of_two_levels_back_read_directly(q4):
    # level 2 reads A's y (level 0) directly while level 1 reads A only through its parts:
    # A's sums must be in y before level 2 waits for them (level 1 writes them at its start)
    import torch

    rng = np.random.default_rng(37)
    h = torch.from_numpy(rng.normal(0, 1, 1024).astype(np.float32)).cuda()
    yA = torch.empty(1000, dtype=torch.float32, device="cuda")
    yC = torch.empty(300, dtype=torch.float32, device="cuda")
    spec = [  # name, N, K, level, x
        ("A", 1000, 1024, 0, h),
        ("C", 300, 512, 1, yA[0:512]),   # through A's parts
        ("F", 200, 512, 2, yA[256:768]),  # A's y itself
        ("G", 96, 256, 2, yC[0:256]),    # through C's parts
    ]
    outs = {"A": yA, "C": yC}
    gemvs, host = [], []
    for name, N, K, lvl, x in spec:
        w = rng.normal(0, 1.0 / np.sqrt(K), (N, K)).astype(np.float32)
        p, s, _ = oracle.pack(w, 4, 128)
        y = outs.get(name)
        if y is None:
            y = torch.empty(N, dtype=torch.float32, device="cuda")
        gemvs.append(q4.StackGemv(torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda(), x, y, N, K, 128, lvl))
        host.append((name, lvl, N, K, 128, p, s))
    st = q4.DecodeStack(gemvs, 4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        st.run(status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_all(gemvs, host, 4, "two levels back")
