"""Pins for the oracle: values the pages print, closed forms, invariants and brute force.

None of these tests re-types the oracle's formula and compares it with the
oracle. Each one checks the oracle against something fixed independently:
numbers printed on the pages (tests/golden/pages.json), hand derivations,
exact rational arithmetic (tests/exact.py) or a brute-force search.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads
from tests.exact import exact_dot, nearest_code, rn32

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rms(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.sqrt(np.mean((a - b) ** 2)))


def roundtrip(w, bits, group):
    payload, scales, st = oracle.pack(w, bits, group)
    assert st == oracle.OK
    return payload, scales, oracle.dequant(payload, scales, np.size(w), bits, group)


# --- the eight-weight worked example ------------------------------------------------

def test_eight_weights_steps(golden):
    g = golden["eight_weights"]
    w = np.array(g["weights"], np.float32)
    _, s8, _ = oracle.pack(w, 8, 8)
    _, s4, _ = oracle.pack(w, 4, 8)
    assert round(float(s8[0]), 6) == g["int8_step_printed"]
    assert round(float(s4[0]), 6) == g["int4_step_printed"]


def test_eight_weights_codes_and_bytes(golden):
    g = golden["eight_weights"]
    w = np.array(g["weights"], np.float32)
    for bits in (8, 4):
        payload, _, codes, st = oracle.pack(w, bits, 8, with_codes=True)
        assert st == oracle.OK
        assert codes.tolist() == g[f"int{bits}_codes_by_hand"]
        assert payload.tolist() == g[f"int{bits}_bytes_by_hand"]
        assert oracle.unpack_codes(payload, 8, bits).tolist() == g[f"int{bits}_codes_by_hand"]


def test_eight_weights_rms_ratio(golden):
    g = golden["eight_weights"]
    w = np.array(g["weights"], np.float32)
    _, _, d8 = roundtrip(w, 8, 8)
    _, _, d4 = roundtrip(w, 4, 8)
    assert round(rms(w, d4) / rms(w, d8), 1) == g["rms_ratio_printed"]


def test_outlier_example(golden):
    g = golden["eight_weights"]
    o = golden["outlier"]
    clean = np.array(g["weights"], np.float32)
    row = np.array(g["weights"] + [o["extra_weight"]], np.float32)
    _, s_clean, _ = roundtrip(clean, 8, 8)
    _, s_out, deq = roundtrip(row, 8, 9)
    assert round(float(s_out[0] / s_clean[0]), 1) == o["coarser_printed"]
    w64 = row.astype(np.float64)
    pct = 100 * np.abs(w64 - deq) / np.abs(w64)
    assert round(float(pct[-1]), 2) == o["outlier_error_pct_printed"]
    assert round(float(pct[:-1].max()), 2) == o["worst_small_error_pct_printed"]


def test_two_scales_example(golden):
    g = golden["eight_weights"]
    o = golden["outlier"]
    row = np.array(g["weights"] + [o["extra_weight"]], np.float32)
    _, _, deq_one = roundtrip(row, 8, 9)
    _, _, deq_a = roundtrip(row[:8], 8, 8)
    _, _, deq_b = roundtrip(row[8:], 8, 1)
    deq_two = np.concatenate([deq_a, deq_b])
    assert round(rms(row, deq_one) / rms(row, deq_two)) == golden["two_scales"]["improvement_printed"]


def test_memory_table(golden):
    m = golden["memory_7b"]
    assert oracle.payload_len(m["params"], 8) / 1e9 == m["int8_gb_printed"]
    assert oracle.payload_len(m["params"], 4) / 1e9 == m["int4_gb_printed"]


# --- pack()'s own checks ------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_pack_checks_roundtrip(golden, bits):
    c = golden["pack_checks"]
    shape = tuple(c["shape"])
    n = shape[0] * shape[1]
    for w in (np.zeros(shape, np.float32), np.linspace(-3, 3, n, dtype=np.float32).reshape(shape)):
        payload, scales, codes, st = oracle.pack(w, bits, c["group"], with_codes=True)
        assert st == oracle.OK
        assert payload.size == n * bits // 8
        expected = (codes.reshape(-1, c["group"]).astype(np.float32) * scales[:, None]).reshape(-1)
        got = oracle.dequant(payload, scales, n, bits, c["group"])
        assert np.array_equal(got.view(np.uint32), expected.view(np.uint32))
        if not w.any():
            assert np.all(scales == 1.0) and not codes.any()


# --- exact arithmetic: scales, quotients and codes -----------------------------------------

def _check_group_exact(w, bits, group):
    qm = oracle.qmax(bits)
    payload, scales, codes, st = oracle.pack(w, bits, group, with_codes=True)
    flat = np.asarray(w, np.float32).reshape(-1)
    for j in range(flat.size // group):
        seg = flat[j * group:(j + 1) * group]
        absmax = max(Fraction(float(abs(v))) for v in seg)
        s = rn32(absmax / qm)
        if s == 0:
            s = np.float32(1.0)
        assert scales[j].view(np.uint32) == np.float32(s).view(np.uint32), (j, scales[j], s)
        for i, v in enumerate(seg):
            t = rn32(Fraction(float(v)) / Fraction(float(s)))
            assert codes[j * group + i] == nearest_code(t, qm)
    return payload, scales, codes


@pytest.mark.parametrize("bits,group", [(4, 16), (8, 16), (4, 32), (8, 48)])
def test_codes_brute_force_adversarial(bits, group):
    rows = workloads.adversarial_rows(96)
    _check_group_exact(rows, bits, group)


def test_codes_brute_force_random():
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, 4 * 64).astype(np.float32)
    for bits in (4, 8):
        _check_group_exact(w, bits, 64)


def test_ties_round_to_even():
    rows = workloads.adversarial_rows(64)
    for bits, row in ((4, rows[2]), (8, rows[3])):
        qm = oracle.qmax(bits)
        _, scales, codes, _ = oracle.pack(row, bits, 16, with_codes=True)
        step = 2.0 ** -4 if bits == 4 else 2.0 ** -8
        assert np.all(scales == np.float32(step))
        q = row.astype(np.float64) / step
        half = np.abs(q - np.floor(q) - 0.5) == 0
        assert half.sum() > 0
        # a tie goes to the even neighbour: both neighbours are k and k+1, pick the even one
        lo = np.floor(q[half]).astype(int)
        expect = np.where(lo % 2 == 0, lo, lo + 1)
        assert np.array_equal(codes[half].astype(int), np.clip(expect, -qm, qm))


def test_underflowing_step_becomes_one():
    rows = workloads.adversarial_rows(64)
    _, scales, codes, _ = oracle.pack(rows[5], 4, 16, with_codes=True)
    assert np.all(scales == 1.0) and not codes.any()


def test_nonfinite_is_flagged():
    w = np.zeros(64, np.float32)
    w[3] = np.inf
    assert oracle.pack(w, 4, 32)[2] == oracle.ERR_NONFINITE
    w[3] = np.nan
    assert oracle.pack(w, 8, 32)[2] == oracle.ERR_NONFINITE


# --- invariants from "Huit bits, puis quatre", section "Arrondir" -------------------------------

@pytest.mark.parametrize("bits,group", [(8, 1024), (4, 32), (4, 128), (8, 128)])
def test_half_step_bound_and_extremal_code(bits, group):
    m = workloads.Matrix("W", 64, 1024, 0.05, 0, 0.001)
    w = workloads.weight(m)
    qm = oracle.qmax(bits)
    payload, scales, codes, _ = oracle.pack(w, bits, group, with_codes=True)
    deq = oracle.dequant(payload, scales, w.size, bits, group)
    s = np.repeat(scales.astype(np.float64), group)
    err = np.abs(w.reshape(-1).astype(np.float64) - deq.astype(np.float64))
    # half a step, plus the rounding of the quotient and of code*scale (a few fp32 ulps)
    assert np.all(err <= 0.5 * s * (1 + 2.0 ** -20) + np.abs(deq) * 2.0 ** -23)
    g = np.abs(w.reshape(-1, group))
    am = g.argmax(axis=1)
    assert np.all(np.abs(codes.reshape(-1, group)[np.arange(g.shape[0]), am]) == qm)


def test_per_row_error_figures(golden):
    p = golden["per_row_1024"]
    w = workloads.weight(workloads.WORKLOADS["small"].matrices[0])
    assert w.shape == (1024, 1024)
    errs = {}
    for bits in (8, 4):
        payload, scales, deq = roundtrip(w, bits, 1024)
        errs[bits] = np.abs(w - deq.reshape(w.shape)).mean() / np.abs(w).mean()
        assert round(payload.size / 1e6, 2) == p[f"int{bits}_mb_printed"]
    assert round(w.nbytes / 1e6, 2) == p["fp32_mb_printed"]
    assert errs[8] < p["int8_mean_rel_err_below"]
    assert round(100 * errs[4]) == p["int4_mean_rel_err_pct_printed"]


def test_groups_may_cross_rows():
    # pack() reshapes the flat tensor to (-1, group): a group may span rows
    rng = np.random.default_rng(7)
    w = rng.normal(0, 1, (6, 40)).astype(np.float32)
    for bits, group in ((4, 48), (8, 240), (4, 240)):
        payload, scales, codes = _check_group_exact(w, bits, group)
        n = w.size
        assert np.array_equal(oracle.unpack_codes(payload, n, bits), codes)
        full = oracle.dequant_rows(payload, scales, 6, 40, bits, group)
        part = oracle.dequant_rows(payload, scales, 6, 40, bits, group, rows=[4, 1])
        assert np.array_equal(part, full[[4, 1]])
        assert np.array_equal(full.reshape(-1), (codes.astype(np.float32).reshape(-1, group) * scales[:, None]).reshape(-1))


def test_dequant_exact_for_power_of_two_steps():
    rows = workloads.adversarial_rows(64)
    payload, scales, codes, _ = oracle.pack(rows[2], 4, 16, with_codes=True)
    deq = oracle.dequant(payload, scales, 64, 4, 16)
    for c, d in zip(codes, deq):
        assert Fraction(float(d)) == Fraction(int(c)) * Fraction(1, 16)


# --- the matmul -----------------------------------------------------------------------------------

def test_matmul_exact_rational_non_square():
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 7
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    w = rng.normal(0, 1, (N, K)).astype(np.float32)
    y, b = oracle.matmul(x, w)
    assert y.shape == (M, N)
    for m in range(M):
        for n in range(N):
            ex = exact_dot(w[n], x[m])
            mag = sum(abs(Fraction(float(a)) * Fraction(float(c))) for a, c in zip(w[n], x[m]))
            assert abs(Fraction(y[m, n]) - ex) <= mag * Fraction(K, 2 ** 52)
            assert abs(Fraction(b[m, n]) - mag) <= mag * Fraction(K, 2 ** 52)


def test_matmul_one_hot_selects_a_weight():
    rng = np.random.default_rng(12)
    N, K = 9, 64
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    payload, scales, st = oracle.pack(w, 4, 32)
    deq = oracle.dequant_rows(payload, scales, N, K, 4, 32)
    for k in (0, 17, 63):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y, _ = oracle.qgemm(x, payload, scales, N, K, 4, 32)
        assert np.array_equal(y[0], deq[:, k].astype(np.float64))


def test_qgemm_integer_weights_exact():
    # every group holds +-7 so the int4 step is exactly 1 and the codes are the weights
    rng = np.random.default_rng(13)
    N, K, g = 4, 32, 16
    codes = rng.integers(-7, 8, (N, K))
    codes[:, ::g] = 7
    w = codes.astype(np.float32)
    x = rng.integers(-50, 50, (2, K)).astype(np.float32)
    payload, scales, st = oracle.pack(w, 4, g)
    assert np.all(scales == 1.0)
    y, _ = oracle.qgemm(x, payload, scales, N, K, 4, g)
    assert np.array_equal(y, (x.astype(np.int64) @ codes.T).astype(np.float64))


def test_qgemm_rows_subset_matches_full():
    rng = np.random.default_rng(14)
    N, K = 12, 256
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = rng.normal(0, 1, (3, K)).astype(np.float32)
    for bits, g in ((4, 128), (8, 256), (4, 64)):
        payload, scales, _ = oracle.pack(w, bits, g)
        y, b = oracle.qgemm(x, payload, scales, N, K, bits, g)
        ys, bs = oracle.qgemm(x, payload, scales, N, K, bits, g, rows=[11, 0, 5])
        assert np.array_equal(ys, y[:, [11, 0, 5]]) and np.array_equal(bs, b[:, [11, 0, 5]])
