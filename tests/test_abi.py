"""The C ABI without a GPU: the library loads, exports every declared symbol, sizes
buffers, and rejects bad arguments on the host before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q4():
    from int4_quantized_b200 import _build

    _build.build()
    import int4_quantized_b200 as m

    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "q4.h")).read()
    return re.findall(r"^Q4_API\s[^;(]*?\b(\w+)\s*\(", src, re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"qpack", "qdequant", "qgemm", "q4_payload_bytes", "q4_num_scales",
            "q4_qgemm_workspace_bytes", "q4_status_str", "q4_version"} <= names


def test_every_declared_symbol_is_exported(q4):
    lib = q4.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_sizes(q4):
    assert q4.payload_bytes(4096, 4096, 4) == 4096 * 4096 // 2
    assert q4.payload_bytes(4096, 4096, 8) == 4096 * 4096
    assert q4.payload_bytes(3, 3, 4) == 0          # odd count cannot be nibble-paired
    assert q4.payload_bytes(-1, 3, 8) == 0
    assert q4.payload_bytes(1, 8, 5) == 0
    assert q4.num_scales(11008, 4096, 128) == 11008 * 32
    assert q4.num_scales(2, 3, 4) == -1
    assert q4.num_scales(2, 3, 0) == -1
    assert q4.lib().q4_version() >= 100


def test_status_strings(q4):
    for code in range(6):
        assert q4.lib().q4_status_str(code)
    assert q4.lib().q4_status_str(99) == b"unknown status"


FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("rows,cols,bits,group,ptr_ok,expect", [
    (4, 32, 3, 32, True, 1),        # bits
    (4, 32, 4, 0, True, 1),         # group
    (4, 32, 4, 48, True, 1),        # group does not divide n
    (1, 3, 4, 3, True, 1),          # odd n for int4
    (-1, 32, 8, 32, True, 1),       # negative size
    (4, 32, 8, 32, False, 1),       # null pointers
    (0, 32, 8, 32, False, 0),       # empty: nothing to do, no pointer needed
])
def test_qpack_validation(q4, rows, cols, bits, group, ptr_ok, expect):
    p = FAKE if ptr_ok else None
    assert q4.lib().qpack(p, rows, cols, bits, group, p, p, None, None) == expect
    assert q4.lib().qdequant(p, p, rows, cols, bits, group, p, None) == expect


@pytest.mark.parametrize("M,N,K,bits,group,xt,expect", [
    (1, 64, 128, 3, 128, 0, 1),     # bits
    (1, 64, 128, 4, 0, 0, 1),       # group
    (1, 64, 128, 4, 128, 7, 1),     # x dtype
    (1, 64, 96, 4, 5, 0, 1),        # group does not divide N * K
    (1, 3, 3, 4, 3, 0, 1),          # an odd number of int4 weights
    (1, 64, 128, 4, 128 * 65, 0, 1),  # whole-row groups that do not divide N
    (65535 * 16 + 1, 64, 128, 4, 128, 0, 2),  # more rows of x than the fused GEMV takes
    (-1, 64, 128, 4, 128, 0, 1),    # negative M
])
def test_qgemm_validation(q4, M, N, K, bits, group, xt, expect):
    assert q4.lib().qgemm(FAKE, xt, M, FAKE, FAKE, N, K, bits, group, FAKE, FAKE, 1 << 30, None, None) == expect


def test_qgemm_workspace_rules(q4):
    lib = q4.lib()
    # 11008 rows: two CTAs per SM, so the pieces of several rows come from the workspace
    need = lib.q4_qgemm_workspace_bytes(8, 11008, 4096, 4, 128, 0)
    assert need > 0 and need % 256 == 0
    # one row of x needs less fragment space than four
    assert lib.q4_qgemm_workspace_bytes(1, 11008, 4096, 4, 128, 0) < lib.q4_qgemm_workspace_bytes(4, 11008, 4096, 4, 128, 0)
    # 4096 rows, one CTA per SM: up to four fp32 rows (and one bf16 row) are built on chip
    for m in (1, 2, 3, 4):
        assert lib.q4_qgemm_workspace_bytes(m, 4096, 4096, 4, 128, 0) == 0
    assert lib.q4_qgemm_workspace_bytes(5, 4096, 4096, 4, 128, 0) > 0
    assert lib.q4_qgemm_workspace_bytes(2, 4096, 4096, 4, 128, 1) > 0  # bf16 rows: from the workspace
    ok = ctypes.c_void_p(0x100000)
    assert lib.qgemm(FAKE, 0, 8, FAKE, FAKE, 11008, 4096, 4, 128, FAKE, None, need, None, None) == 5
    assert lib.qgemm(FAKE, 0, 8, FAKE, FAKE, 11008, 4096, 4, 128, FAKE, ok, need - 1, None, None) == 5
    assert lib.qgemm(FAKE, 0, 8, FAKE, FAKE, 11008, 4096, 4, 128, FAKE, ctypes.c_void_p(0x100010), need, None, None) == 5
    # misaligned payload / x are reported before anything is enqueued
    assert lib.qgemm(FAKE, 0, 8, ctypes.c_void_p(0x100001), FAKE, 4096, 4096, 4, 128, FAKE, ok, need, None, None) == 2
    assert lib.qgemm(ctypes.c_void_p(0x100004), 0, 8, FAKE, FAKE, 4096, 4096, 4, 128, FAKE, ok, need, None, None) == 2
    # an empty problem enqueues nothing and needs no pointers
    assert lib.qgemm(None, 0, 0, None, None, 4096, 4096, 4, 128, None, None, 0, None, None) == 0
    assert lib.qgemm(None, 0, 8, None, None, 0, 4096, 4, 128, None, None, 0, None, None) == 0


def test_qgemm_ex_flags_and_limits(q4):
    lib = q4.lib()
    ok = ctypes.c_void_p(0x100000)
    need = lib.q4_qgemm_workspace_bytes(8, 11008, 4096, 4, 128, 0)  # two CTAs per SM: a workspace
    # unknown flag bits are refused before anything else is looked at
    for flags in (2, 4, 0x80000000):
        assert lib.qgemm_ex(FAKE, 0, 8, FAKE, FAKE, 4096, 4096, 4, 128, FAKE, ok, need, flags, None, None) == 1
    # with the static-weights flag the argument rules are those of qgemm
    assert lib.qgemm_ex(FAKE, 0, 65535 * 16 + 1, FAKE, FAKE, 64, 128, 4, 128, FAKE, None, 0, 1, None, None) == 2
    assert lib.qgemm_ex(FAKE, 0, 1, FAKE, FAKE, 64, 128, 4, 5, FAKE, None, 0, 1, None, None) == 1
    assert lib.qgemm_ex(FAKE, 0, 8, FAKE, FAKE, 11008, 4096, 4, 128, FAKE, None, need, 1, None, None) == 5
    assert lib.qgemm_ex(None, 0, 0, None, None, 4096, 4096, 4, 128, None, None, 0, 1, None, None) == 0
    # rows of x: at most 65535 chunks of 16
    assert q4.qgemm_workspace_bytes(65535 * 16, 256, 1024, 4, 128) > 0
    assert lib.qgemm(FAKE, 0, 65535 * 16 + 1, FAKE, FAKE, 256, 1024, 4, 128, FAKE, ok, 1 << 40, None, None) == 2


def test_groups_of_whole_rows(q4):
    import torch

    lib = q4.lib()
    N, K = 64, 256
    # one scale for the whole matrix, and groups of 2 and 4 rows: N floats of spread scales
    for g in (N * K, 2 * K, 4 * K):
        assert q4.qgemm_workspace_bytes(1, N, K, 4, g) == 256
        assert q4.qgemm_workspace_bytes(300, N, K, 4, g, torch.bfloat16) == 256  # the GEMM needs only those
        assert q4.qgemm_workspace_bytes(8, N, K, 8, g) == 256 + q4.qgemm_workspace_bytes(8, N, K, 8, K)
    assert q4.qgemm_workspace_bytes(1, 1000, K, 4, K * 1000) == 4096
    # groups that do not divide N * K: no packed tensor has them
    ok = ctypes.c_void_p(0x100000)
    assert lib.qgemm(FAKE, 0, 1, FAKE, FAKE, N, K, 4, 3 * K // 2, FAKE, ok, 1 << 20, None, None) == 1
    assert lib.qgemm(FAKE, 0, 1, FAKE, FAKE, 63, K, 4, 2 * K, FAKE, ok, 1 << 20, None, None) == 1
    # the spread scales must fit in the workspace
    assert lib.qgemm(FAKE, 0, 1, FAKE, FAKE, N, K, 4, N * K, FAKE, ok, 255, None, None) == 5
    assert lib.qgemm(FAKE, 0, 1, FAKE, FAKE, N, K, 4, N * K, FAKE, None, 0, None, None) == 5


def test_workspace_is_a_pure_function_of_the_problem(q4):
    for M in (1, 4, 8, 16, 40, 300, 2048):
        a = q4.qgemm_workspace_bytes(M, 11008, 4096, 4, 128)
        b = q4.qgemm_workspace_bytes(M, 11008, 4096, 4, 128)
        assert a == b and a % 256 == 0


def test_any_group_is_planned(q4):
    # every group qpack accepts plans (M = 0 returns Q4_OK only after the plan accepted the
    # shape): narrow groups dividing K, groups crossing rows at varying offsets, odd K; the
    # any-group path needs no workspace
    import torch

    lib = q4.lib()
    for N, K, bits, g in [(64, 256, 4, 16), (96, 256, 8, 48), (66, 256, 4, 384), (30, 77, 4, 10),
                          (7, 3, 8, 7), (33, 100, 4, 50), (64, 96, 4, 1), (12, 100, 8, 100)]:
        assert lib.qgemm(None, 0, 0, None, None, N, K, bits, g, None, None, 0, None, None) == 0, (N, K, g)
        assert q4.qgemm_workspace_bytes(1, N, K, bits, g) == 0
        assert q4.qgemm_workspace_bytes(100, N, K, bits, g, torch.bfloat16) == 0
    # not a divisor of N * K, or an odd number of int4 weights: no such payload
    assert lib.qgemm(None, 0, 0, None, None, 30, 77, 4, 4, None, None, 0, None, None) == 1
    assert lib.qgemm(None, 0, 0, None, None, 7, 3, 4, 7, None, None, 0, None, None) == 1
    assert lib.qgemm(None, 0, 0, None, None, 7, 3, 8, 7, None, None, 0, None, None) == 0
