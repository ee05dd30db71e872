"""qpack / qdequant on the GPU vs the oracle: payload bytes, scales and dequantized
weights must be bit-identical (pack()/unpack() of the "量化推理" page)."""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    import torch  # noqa: F401

    import int4_quantized_b200 as m

    m.lib()
    return m


def gpu_pack(q4, w, bits, group, status=False):
    import torch

    wt = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if status else None
    payload, scales = q4.qpack(wt.reshape(w.shape[0] if w.ndim else 1, -1), bits, group, status=st)
    torch.cuda.synchronize()
    out = payload.cpu().numpy(), scales.cpu().numpy()
    return (out + (int(st.item()),)) if status else out


def assert_same_bits(a, b, what):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    assert a.shape == b.shape, what
    va = a.view(np.uint8) if a.dtype == np.uint8 else a.view(np.uint32)
    vb = b.view(np.uint8) if b.dtype == np.uint8 else b.view(np.uint32)
    bad = np.flatnonzero(va.reshape(-1) != vb.reshape(-1))
    assert bad.size == 0, f"{what}: {bad.size} mismatches, first at {bad[:5]}"


def check_pack(q4, w, bits, group, dequant=True):
    import torch

    payload, scales = gpu_pack(q4, w, bits, group)
    rp, rs, st = oracle.pack(w, bits, group)
    assert st == oracle.OK
    assert_same_bits(scales, rs, f"scales bits={bits} g={group}")
    assert_same_bits(payload, rp, f"payload bits={bits} g={group}")
    if dequant:
        d = q4.qdequant(torch.from_numpy(payload).cuda(), torch.from_numpy(scales).cuda(), w.shape, bits, group)
        rd = oracle.dequant(rp, rs, w.size, bits, group).reshape(w.shape)
        assert_same_bits(d.cpu().numpy(), rd, f"dequant bits={bits} g={group}")


@pytest.mark.parametrize("name", ["small", "mid", "prefill"])
def test_configs_full(q4, name):
    wl = workloads.WORKLOADS[name]
    for m in wl.matrices:
        w = workloads.weight(m)
        for bits, g in wl.formats:
            check_pack(q4, w, bits, m.K if g is None else g)


@pytest.mark.parametrize("idx", [0, 4, 6, 7 * 31 + 2])  # L0.q, L0.gate, L0.down, L31.v
def test_llama7b_matrices(q4, idx):
    wl = workloads.WORKLOADS["llama7b"]
    m = wl.matrices[idx]
    w = workloads.weight(m)
    for bits, g in wl.formats:
        check_pack(q4, w, bits, m.K if g is None else g, dequant=(idx == 0))


@pytest.mark.parametrize("which", [0, 2])
def test_mlp70b_matrices(q4, which):
    wl = workloads.WORKLOADS["mlp70b"]
    m = wl.matrices[which]
    w = workloads.weight(m)
    check_pack(q4, w, 4, 64, dequant=False)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
def test_adversarial_groups(q4, bits, group):
    rows = workloads.adversarial_rows(4096)
    assert rows.size % group == 0
    check_pack(q4, rows, bits, group)


@pytest.mark.parametrize("bits,group,shape", [
    (4, 3, (2, 3)),            # odd group: a byte straddles two groups
    (4, 5, (6, 5)),
    (8, 7, (3, 7)),
    (4, 2, (1, 2)),
    (8, 1, (4, 4)),            # one scale per weight
    (4, 6, (5, 6)),
    (4, 40, (7, 40)),          # group % 16 != 0
    (4, 4096 * 3, (3, 4096)),  # one scale for the whole tensor
    (8, 65536, (2, 32768)),    # group too large for the register-resident kernel
    (4, 96 * 7, (7, 96)),      # groups span rows
])
def test_generic_shapes(q4, bits, group, shape):
    rng = np.random.default_rng(sum(shape) + group)
    w = rng.normal(0, 1, shape).astype(np.float32)
    check_pack(q4, w, bits, group)


def test_ragged_tail(q4):
    # a tensor whose size is not a multiple of the vector kernel's warp chunk
    rng = np.random.default_rng(3)
    for bits, n in ((4, 1024 * 5 + 64), (8, 512 * 3 + 32)):
        w = rng.normal(0, 0.1, (1, n)).astype(np.float32)
        check_pack(q4, w, bits, 32)


def test_misaligned_input(q4):
    import torch

    rng = np.random.default_rng(4)
    w = rng.normal(0, 0.1, (8, 256)).astype(np.float32)
    base = torch.zeros(w.size + 1, dtype=torch.float32, device="cuda")
    base[1:] = torch.from_numpy(w.reshape(-1)).cuda()
    view = base[1:].reshape(8, 256)  # 4-byte aligned only: takes the generic kernels
    for bits in (4, 8):
        payload, scales = q4.qpack(view, bits, 32)
        rp, rs, _ = oracle.pack(w, bits, 32)
        assert_same_bits(payload.cpu().numpy(), rp, "payload")
        assert_same_bits(scales.cpu().numpy(), rs, "scales")


def test_nonfinite_sets_status(q4):
    w = np.zeros((4, 256), np.float32)
    assert gpu_pack(q4, w, 4, 128, status=True)[2] == 0
    w[2, 7] = np.inf
    assert gpu_pack(q4, w, 4, 128, status=True)[2] == q4.STATUS_NONFINITE
    w[2, 7] = np.nan
    assert gpu_pack(q4, w, 8, 256, status=True)[2] == q4.STATUS_NONFINITE
    w = np.zeros((1, 4096 * 2), np.float32)
    w[0, 5000] = -np.inf
    assert gpu_pack(q4, w, 8, 4096 * 2, status=True)[2] == q4.STATUS_NONFINITE


def test_empty(q4):
    import torch

    w = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    p, s = q4.qpack(w, 4, 128)
    assert p.numel() == 0 and s.numel() == 0
