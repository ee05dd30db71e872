"""int4_quantized_b200 -- Python binding of libq4 (include/q4.h), B200 / sm_100a.

Symmetric round-to-nearest weight quantization with one fp32 scale per group of g
consecutive weights (pack()/unpack() of the "量化推理：INT8/INT4 ..." page; "Huit bits,
puis quatre", section "Arrondir"), and the quantized matmul that reads the packed codes.

This module only marshals arguments: it turns torch CUDA tensors into device pointers
and the current CUDA stream into a cudaStream_t, and checks status codes. Every step of
the computation runs in the CUDA kernels of libq4.so. There is no CPU fallback: if the
library is missing or a call is unsupported, an exception is raised.

    payload, scales = qpack(w, bits=4, group=128)           # w: [N, K] float32 CUDA tensor
    w_deq = qdequant(payload, scales, (N, K), 4, 128)        # float32, bit-exact
    y = qgemm(x, payload, scales, N, K, 4, 128)              # x: [M, K] fp32 or bf16 -> y [M, N]
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "Q4Error", "lib", "lib_path", "payload_bytes", "num_scales", "qgemm_workspace_bytes",
    "qpack", "qdequant", "qgemm", "qgemm_noalloc", "StackGemv", "DecodeStack", "gptq_hessian", "gptq_prepare", "gptq_quantize", "gptq_pack", "NOALLOC_SCRATCH_BYTES", "Q4_OK", "Q4_ERR_ARG", "Q4_ERR_UNSUPPORTED", "Q4_ERR_CUDA",
    "Q4_ERR_NONFINITE", "Q4_ERR_WORKSPACE", "Q4_ERR_SCRATCH_LIMIT", "Q4_X_F32", "Q4_X_BF16", "Q4_QGEMM_WEIGHTS_STATIC", "STATUS_NONFINITE", "STATUS_TIMEOUT",
]

Q4_OK, Q4_ERR_ARG, Q4_ERR_UNSUPPORTED, Q4_ERR_CUDA, Q4_ERR_NONFINITE, Q4_ERR_WORKSPACE, \
    Q4_ERR_SCRATCH_LIMIT = range(7)
NOALLOC_SCRATCH_BYTES = 4 << 20  # Q4_NOALLOC_SCRATCH_BYTES
Q4_X_F32, Q4_X_BF16 = 0, 1
Q4_QGEMM_WEIGHTS_STATIC = 1
STATUS_NONFINITE = 1
STATUS_TIMEOUT = 2

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libq4.so")

_lib = None
_lock = threading.Lock()


class Q4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = f"{what}: {lib().q4_status_str(code).decode()} (status {code})"
        if code == Q4_ERR_CUDA:
            msg += f": {lib().q4_last_cuda_error().decode()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """Load libq4.so (built in-tree by ``python -m int4_quantized_b200._build``)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(lib_path):
                    raise ImportError(
                        f"libq4.so is not built at {lib_path}; run `python -m int4_quantized_b200._build`")
                L = ctypes.CDLL(lib_path)
                i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
                L.q4_version.restype = i32
                L.q4_status_str.argtypes = [i32]
                L.q4_status_str.restype = ctypes.c_char_p
                L.q4_last_cuda_error.restype = ctypes.c_char_p
                L.q4_payload_bytes.argtypes = [i64, i64, i32]
                L.q4_payload_bytes.restype = sz
                L.q4_num_scales.argtypes = [i64, i64, i64]
                L.q4_num_scales.restype = i64
                L.qpack.argtypes = [vp, i64, i64, i32, i64, vp, vp, vp, vp]
                L.qpack.restype = i32
                L.qdequant.argtypes = [vp, vp, i64, i64, i32, i64, vp, vp]
                L.qdequant.restype = i32
                L.q4_qgemm_workspace_bytes.argtypes = [i64, i64, i64, i32, i64, i32]
                L.q4_qgemm_workspace_bytes.restype = sz
                L.qgemm.argtypes = [vp, i32, i64, vp, vp, i64, i64, i32, i64, vp, vp, sz, vp, vp]
                L.qgemm.restype = i32
                L.qgemm_ex.argtypes = [vp, i32, i64, vp, vp, i64, i64, i32, i64, vp, vp, sz, ctypes.c_uint32, vp,
                                       vp]
                L.qgemm_ex.restype = i32
                L.qgemm_noalloc.argtypes = [vp, i32, i64, vp, vp, i64, i64, i32, i64, vp, vp, vp]
                L.qgemm_noalloc.restype = i32
                L.q4_stack_workspace_bytes.argtypes = [vp, ctypes.c_int32, i32, i32]
                L.q4_stack_workspace_bytes.restype = sz
                L.q4_stack_prepare.argtypes = [vp, ctypes.c_int32, i32, i32, vp, sz, vp, vp]
                L.q4_stack_prepare.restype = i32
                L.q4_stack_run.argtypes = [vp, vp, vp]
                L.q4_stack_run.restype = i32
                L.q4_stack_set_wait_limit.argtypes = [vp, ctypes.c_uint64]
                L.q4_stack_set_wait_limit.restype = i32
                L.q4_gptq_hessian.argtypes = [vp, i64, i64, vp, i32]
                L.q4_gptq_hessian.restype = i32
                L.q4_gptq_prepare.argtypes = [vp, i64, ctypes.c_double, vp, i32]
                L.q4_gptq_prepare.restype = i32
                L.q4_gptq_quantize.argtypes = [vp, i64, i64, vp, i32, i64, vp, vp, i32]
                L.q4_gptq_quantize.restype = i32
                _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(code: int, what: str):
    if code != Q4_OK:
        raise Q4Error(code, what)


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def payload_bytes(rows: int, cols: int, bits: int) -> int:
    return int(lib().q4_payload_bytes(rows, cols, bits))


def num_scales(rows: int, cols: int, group: int) -> int:
    return int(lib().q4_num_scales(rows, cols, group))


def qgemm_workspace_bytes(M: int, N: int, K: int, bits: int, group: int, x_dtype=torch.float32) -> int:
    xt = Q4_X_BF16 if x_dtype == torch.bfloat16 else Q4_X_F32
    return int(lib().q4_qgemm_workspace_bytes(M, N, K, bits, group, xt))


def qpack(w: torch.Tensor, bits: int, group: int, payload: Optional[torch.Tensor] = None,
          scales: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None
          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Quantize a float32 CUDA tensor (flattened row-major) -> (payload uint8, scales float32)."""
    _cuda(w, "w", torch.float32)
    rows = w.shape[0] if w.dim() >= 1 else 1
    cols = w.numel() // rows if rows else 0
    nb = payload_bytes(rows, cols, bits)
    ns = num_scales(rows, cols, group)
    if payload is None:
        payload = torch.empty(nb, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(max(ns, 0), dtype=torch.float32, device=w.device)
    if status is not None:
        _cuda(status, "status", torch.int32)
    with torch.cuda.device(w.device):
        _check(lib().qpack(_ptr(w), rows, cols, bits, group, _ptr(payload), _ptr(scales),
                           _ptr(status), _stream(w.device)), "qpack")
    return payload, scales


def qdequant(payload: torch.Tensor, scales: torch.Tensor, shape: Sequence[int], bits: int, group: int,
             out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Decode packed codes -> float32 tensor of `shape` (code * scale, bit-exact)."""
    _cuda(payload, "payload", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    shape = tuple(int(s) for s in shape)
    rows = shape[0] if shape else 1
    n = 1
    for s in shape:
        n *= s
    cols = n // rows if rows else 0
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=payload.device)
    with torch.cuda.device(payload.device):
        _check(lib().qdequant(_ptr(payload), _ptr(scales), rows, cols, bits, group, _ptr(out),
                              _stream(payload.device)), "qdequant")
    return out


_ws_cache = {}


def _workspace(dev: torch.device, nbytes: int) -> torch.Tensor:
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


def qgemm(x: torch.Tensor, payload: torch.Tensor, scales: torch.Tensor, N: int, K: int, bits: int,
          group: int, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
          status: Optional[torch.Tensor] = None, weights_static: bool = False) -> torch.Tensor:
    """y[M, N] = x[M, K] @ W'^T from the packed codes (x float32 or bfloat16).

    weights_static=True (Q4_QGEMM_WEIGHTS_STATIC): payload and scales may be streamed
    while the previous kernel on the stream still runs; only valid when their last write
    finished before that kernel started (weights packed once, then reused).
    """
    _cuda(x, "x")
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _cuda(payload, "payload", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    x2 = x.reshape(-1, K)
    M = x2.shape[0]
    xt = Q4_X_BF16 if x.dtype == torch.bfloat16 else Q4_X_F32
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    else:
        _cuda(out, "out", torch.float32)
    need = int(lib().q4_qgemm_workspace_bytes(M, N, K, bits, group, xt))
    if workspace is None and need > 0:
        workspace = _workspace(x.device, need)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if status is not None:
        _cuda(status, "status", torch.int32)
    with torch.cuda.device(x.device):
        _check(lib().qgemm_ex(_ptr(x2), xt, M, _ptr(payload), _ptr(scales), N, K, bits, group, _ptr(out),
                              _ptr(workspace), ws_bytes, Q4_QGEMM_WEIGHTS_STATIC if weights_static else 0,
                              _ptr(status), _stream(x.device)), "qgemm")
    return out


def qgemm_noalloc(x: torch.Tensor, payload: torch.Tensor, scales: torch.Tensor, N: int, K: int,
                  bits: int, group: int, out: torch.Tensor, status: Optional[torch.Tensor] = None
                  ) -> torch.Tensor:
    """qgemm into a caller-given `out` using the library's built-in device scratch.

    Allocates nothing. All calls on one device share that scratch, so calls that may
    overlap on the GPU race; calls on one stream are safe.
    """
    _cuda(x, "x")
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _cuda(payload, "payload", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    _cuda(out, "out", torch.float32)
    M = x.numel() // K if K else 0
    xt = Q4_X_BF16 if x.dtype == torch.bfloat16 else Q4_X_F32
    if status is not None:
        _cuda(status, "status", torch.int32)
    with torch.cuda.device(x.device):
        _check(lib().qgemm_noalloc(_ptr(x), xt, M, _ptr(payload), _ptr(scales), N, K, bits, group,
                                   _ptr(out), _ptr(status), _stream(x.device)), "qgemm_noalloc")
    return out


# ---- decode stack: every GEMV of a decode step in one persistent kernel -----------------

class _StackGemvC(ctypes.Structure):
    _fields_ = [("payload", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("group", ctypes.c_int64),
                ("level", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class StackGemv:
    """One GEMV of a decode stack: y[N] = W'[N, K] x[K] (x float32 or bfloat16)."""

    def __init__(self, payload: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, y: torch.Tensor,
                 N: int, K: int, group: int, level: int):
        _cuda(payload, "payload", torch.uint8)
        _cuda(scales, "scales", torch.float32)
        _cuda(x, "x")
        _cuda(y, "y", torch.float32)
        if x.numel() != K or y.numel() != N:
            raise ValueError("x must hold K values and y N values")
        self.payload, self.scales, self.x, self.y = payload, scales, x, y
        self.N, self.K, self.group, self.level = int(N), int(K), int(group), int(level)


class DecodeStack:
    """A prepared stack of GEMVs (q4_stack_prepare); run() is one launch of all of them.

    Levels: the GEMVs of level l may read what GEMVs of earlier levels write; every GEMV
    of level l - 1 has finished writing before level l reads its x. The workspace and the
    tensors of every GEMV are held for the life of the object.
    """

    def __init__(self, gemvs: Sequence[StackGemv], bits: int):
        if not gemvs:
            raise ValueError("empty stack")
        dt = gemvs[0].x.dtype
        if dt not in (torch.float32, torch.bfloat16) or any(g.x.dtype != dt for g in gemvs):
            raise TypeError("every x must have the same dtype, float32 or bfloat16")
        self.gemvs = list(gemvs)
        self.bits = bits
        self.device = gemvs[0].payload.device
        xt = Q4_X_BF16 if dt == torch.bfloat16 else Q4_X_F32
        arr = (_StackGemvC * len(gemvs))()
        for i, g in enumerate(gemvs):
            arr[i] = _StackGemvC(g.payload.data_ptr(), g.scales.data_ptr(), g.x.data_ptr(), g.y.data_ptr(),
                                 g.N, g.K, g.group, g.level, 0)
        n = len(gemvs)
        need = int(lib().q4_stack_workspace_bytes(ctypes.byref(arr), n, bits, xt))
        if need == 0:
            raise Q4Error(Q4_ERR_ARG, "stack_workspace_bytes")
        self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        self._plan = (ctypes.c_uint64 * 32)()
        with torch.cuda.device(self.device):
            _check(lib().q4_stack_prepare(ctypes.byref(arr), n, bits, xt, _ptr(self.workspace), need,
                                          ctypes.byref(self._plan), _stream(self.device)), "stack_prepare")
        self.weight_bytes = sum(g.payload.numel() + 4 * g.scales.numel() for g in gemvs)

    def set_wait_limit(self, nanoseconds: int) -> None:
        """Bound of every wait inside the kernel (default 1e9 ns); see q4_stack_set_wait_limit."""
        _check(lib().q4_stack_set_wait_limit(ctypes.byref(self._plan), int(nanoseconds)), "stack_set_wait_limit")

    def run(self, status: Optional[torch.Tensor] = None) -> None:
        if status is not None:
            _cuda(status, "status", torch.int32)
        with torch.cuda.device(self.device):
            _check(lib().q4_stack_run(ctypes.byref(self._plan), _ptr(status), _stream(self.device)), "stack_run")


# ---- GPTQ host quantizer (host arrays; the computation runs in libq4's C++ code) ----------

def _host(a, dtype, name):
    import numpy as np

    if isinstance(a, torch.Tensor):
        if a.is_cuda:
            raise TypeError(f"{name} must be host memory (a NumPy array or a CPU tensor)")
        a = a.numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"{name} must be {np.dtype(dtype).name}, got {a.dtype}")
    return a


def gptq_hessian(x, H=None, threads: int = 0):
    """H += x^T x in fp64 for calibration inputs x [rows, K] float32 (H new when None)."""
    import numpy as np

    x = _host(x, np.float32, "x")
    rows, K = x.shape
    if H is None:
        H = np.zeros((K, K), np.float64)
    elif not (isinstance(H, np.ndarray) and H.dtype == np.float64 and H.shape == (K, K) and H.flags.c_contiguous):
        raise TypeError("H must be a C-contiguous float64 [K, K] NumPy array")
    _check(lib().q4_gptq_hessian(x.ctypes.data_as(ctypes.c_void_p), rows, K, H.ctypes.data_as(ctypes.c_void_p),
                                 threads), "gptq_hessian")
    return H


def gptq_prepare(H, damp: float = 0.01, threads: int = 0):
    """U (upper, fp64) with (H + damp * mean(diag H) * I)^-1 = U^T U."""
    import numpy as np

    H = _host(H, np.float64, "H")
    K = H.shape[0]
    U = np.empty((K, K), np.float64)
    _check(lib().q4_gptq_prepare(H.ctypes.data_as(ctypes.c_void_p), K, damp, U.ctypes.data_as(ctypes.c_void_p),
                                 threads), "gptq_prepare")
    return U


def gptq_quantize(w, U, bits: int, group: int, threads: int = 0):
    """(payload uint8, scales float32) of W [N, K] float32 by GPTQ, in qpack's format."""
    import numpy as np

    w = _host(w, np.float32, "w")
    U = _host(U, np.float64, "U")
    N, K = w.shape
    if U.shape != (K, K):
        raise ValueError("U must be [K, K]")
    payload = np.empty(N * K * bits // 8, np.uint8)
    scales = np.empty(N * K // group if group > 0 and K % group == 0 else 0, np.float32)
    _check(lib().q4_gptq_quantize(w.ctypes.data_as(ctypes.c_void_p), N, K, U.ctypes.data_as(ctypes.c_void_p), bits,
                                  group, payload.ctypes.data_as(ctypes.c_void_p),
                                  scales.ctypes.data_as(ctypes.c_void_p), threads), "gptq_quantize")
    return payload, scales


def gptq_pack(w, x, bits: int, group: int, damp: float = 0.01, threads: int = 0):
    """GPTQ end to end on the host: H from calibration inputs x [rows, K], then the codes."""
    H = gptq_hessian(x, threads=threads)
    return gptq_quantize(w, gptq_prepare(H, damp, threads), bits, group, threads)
