"""Python access to the oracle (qref.c) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The
product path (``int4_quantized_b200``) never imports it and has no CPU
fallback.

The C file states what each function follows on the pages (pack()/unpack() of
the "量化推理：INT8/INT4 ..." page, the rule of "Huit bits, puis quatre",
section "Arrondir"). This wrapper only marshals NumPy arrays; it adds no
arithmetic of its own except selecting which rows to decode for a sampled
matmul.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qref.c")
_LIB = os.path.join(_HERE, "libqref.so")

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c99"]

OK, ERR_ARG, ERR_NONFINITE = 0, 1, 4


def build(force: bool = False) -> str:
    """Compile qref.c into libqref.so with gcc (no CUDA involved)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.qref_qmax.argtypes = [i32]
        lib.qref_pack.argtypes = [vp, i64, i32, i64, vp, vp, vp]
        lib.qref_unpack_codes.argtypes = [vp, i64, i32, vp]
        lib.qref_dequant.argtypes = [vp, vp, i64, i32, i64, i64, vp]
        lib.qref_matmul.argtypes = [vp, i64, vp, i64, i64, vp, vp]
        for f in (lib.qref_pack, lib.qref_unpack_codes, lib.qref_dequant, lib.qref_matmul, lib.qref_qmax):
            f.restype = i32
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def qmax(bits: int) -> int:
    return int(_load().qref_qmax(bits))


def payload_len(n: int, bits: int) -> int:
    return n * bits // 8


def pack(w: np.ndarray, bits: int, group: int, with_codes: bool = False):
    """pack(w, bits, group) -> (payload uint8, scales float32[, codes int8], status).

    The array is flattened row-major, as pack() reshapes to (-1, group).
    """
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    n = w.size
    if group < 1 or n % group:
        raise ValueError("group must divide the number of weights")
    payload = np.zeros(payload_len(n, bits), np.uint8)
    scales = np.zeros(n // group, np.float32)
    codes = np.zeros(n, np.int8) if with_codes else None
    st = _load().qref_pack(_ptr(w), n, bits, group, _ptr(payload), _ptr(scales), _ptr(codes))
    if st == ERR_ARG:
        raise ValueError("qref_pack rejected its arguments")
    if with_codes:
        return payload, scales, codes, st
    return payload, scales, st


def unpack_codes(payload: np.ndarray, n: int, bits: int) -> np.ndarray:
    payload = np.ascontiguousarray(payload, dtype=np.uint8)
    codes = np.zeros(n, np.int8)
    if _load().qref_unpack_codes(_ptr(payload), n, bits, _ptr(codes)) != OK:
        raise ValueError("qref_unpack_codes rejected its arguments")
    return codes


def dequant(payload: np.ndarray, scales: np.ndarray, n: int, bits: int, group: int,
            base_index: int = 0) -> np.ndarray:
    """w' (float32, flat) for `n` weights starting at flat index `base_index`.

    `payload` is the slice holding those n weights; `scales` is the full scale
    array of the tensor.
    """
    payload = np.ascontiguousarray(payload, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    out = np.zeros(n, np.float32)
    if _load().qref_dequant(_ptr(payload), _ptr(scales), n, bits, group, base_index, _ptr(out)) != OK:
        raise ValueError("qref_dequant rejected its arguments")
    return out


def matmul(x: np.ndarray, w: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """y = x @ w^T accumulated in fp64 (ascending k), and bound = |x| @ |w|^T."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    M, K = x.shape
    N, K2 = w.shape
    assert K == K2
    y = np.zeros((M, N), np.float64)
    b = np.zeros((M, N), np.float64)
    if _load().qref_matmul(_ptr(x), M, _ptr(w), N, K, _ptr(y), _ptr(b)) != OK:
        raise ValueError("qref_matmul rejected its arguments")
    return y, b


def dequant_rows(payload: np.ndarray, scales: np.ndarray, N: int, K: int, bits: int, group: int,
                 rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """W' rows [len(rows), K] (all rows when rows is None)."""
    payload = np.ascontiguousarray(payload, dtype=np.uint8).reshape(-1)
    if rows is None:
        return dequant(payload, scales, N * K, bits, group).reshape(N, K)
    rb = K * bits // 8
    out = np.zeros((len(rows), K), np.float32)
    for i, r in enumerate(rows):
        out[i] = dequant(payload[r * rb:(r + 1) * rb], scales, K, bits, group, base_index=r * K)
    return out


def qgemm(x: np.ndarray, payload: np.ndarray, scales: np.ndarray, N: int, K: int, bits: int,
          group: int, rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """The quantized matmul by its definition: decode W', then y = x W'^T in fp64.

    With `rows`, only those output channels are computed (columns of y).
    """
    w = dequant_rows(payload, scales, N, K, bits, group, rows)
    return matmul(x, w)
