"""qgemm with Q4_QGEMM_WEIGHTS_STATIC (payload and scales streamed while the previous
kernel on the stream still runs): the same bits as the plain call, and stream order kept
for x and y.

The chain test feeds each call's y to the next call as x, and lets each call overwrite
the buffer the call before it read (ping-pong): a read of x that did not wait for the
previous kernel, or a write that overtook its reads, changes the bits of the final y.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import int4_quantized_b200 as m

    m.lib()
    return m


def packed(q4, N, K, bits, group, seed):
    import torch

    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    p, s, _ = oracle.pack(w, bits, group)
    return torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda()


@pytest.mark.parametrize("bits,group", [(4, 128), (8, 4096), (4, 32)])
@pytest.mark.parametrize("M", [1, 3, 16])
def test_same_bits_as_plain_call(q4, bits, group, M):
    import torch

    N, K = 1536, 4096
    P, S = packed(q4, N, K, bits, group, 5 + M)
    x = torch.from_numpy(np.random.default_rng(M).normal(0, 1, (M, K)).astype(np.float32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y0 = q4.qgemm(x, P, S, N, K, bits, group, status=status)
    y1 = q4.qgemm(x, P, S, N, K, bits, group, status=status, weights_static=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))


@pytest.mark.parametrize("M", [1, 4])
def test_chain_keeps_stream_order(q4, M):
    import torch

    K = 4096
    mats = [packed(q4, K, K, 4 if i % 2 == 0 else 8, 128 if i % 2 == 0 else K, 40 + i) for i in range(6)]
    fmt = [(4, 128) if i % 2 == 0 else (8, K) for i in range(6)]
    x0 = torch.from_numpy(np.random.default_rng(2).normal(0, 1, (M, K)).astype(np.float32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def chain(static):
        a, b = x0.clone(), torch.empty_like(x0)
        torch.cuda.synchronize()
        for rep in range(3):
            for (P, S), (bits, g) in zip(mats, fmt):
                q4.qgemm(a, P, S, K, K, bits, g, out=b, status=status, weights_static=static)
                # keep the values in range: the next call reads b, then this scale runs
                # between the calls as an unrelated kernel on the same stream
                b.mul_(0.5)
                a, b = b, a
        torch.cuda.synchronize()
        return a.clone()

    ref = chain(False)
    got = chain(True)
    assert int(status.item()) == 0
    assert torch.all(torch.isfinite(ref))
    assert torch.equal(ref.view(torch.int32), got.view(torch.int32))

    # back to back with no other kernel between the calls
    def chain_direct(static):
        bufs = [x0.clone()] + [torch.empty_like(x0) for _ in range(len(mats))]
        torch.cuda.synchronize()
        for i, ((P, S), (bits, g)) in enumerate(zip(mats, fmt)):
            q4.qgemm(bufs[i], P, S, K, K, bits, g, out=bufs[i + 1], status=status, weights_static=static)
        torch.cuda.synchronize()
        return bufs[-1].clone()

    assert torch.equal(chain_direct(False).view(torch.int32), chain_direct(True).view(torch.int32))
    assert int(status.item()) == 0


def test_ping_pong_without_other_kernels(q4):
    # y of call i is x of call i + 1, and call i + 1 writes the buffer call i read
    import torch

    K = 2048
    P, S = packed(q4, K, K, 4, 128, 77)
    x0 = torch.from_numpy(np.random.default_rng(3).normal(0, 1, (1, K)).astype(np.float32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(static):
        a, b = x0.clone(), torch.empty_like(x0)
        torch.cuda.synchronize()
        for _ in range(12):
            q4.qgemm(a, P, S, K, K, 4, 128, out=b, status=status, weights_static=static)
            a, b = b, a
        torch.cuda.synchronize()
        return a.clone()

    ref, got = run(False), run(True)
    assert int(status.item()) == 0
    assert torch.all(torch.isfinite(ref))
    assert torch.equal(ref.view(torch.int32), got.view(torch.int32))
