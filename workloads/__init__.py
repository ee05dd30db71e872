"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers. It holds none of the quantization or
matmul arithmetic, so both sides can use it without sharing method code.

Every workload is a weight matrix W of shape [N, K] (N output channels, K
inputs, row-major, fp32) plus activation rows x of shape [M, K]. Groups of g
consecutive weights in the row-major flattening share one scale, so with g | K
they run along K inside one row.

Recipes (NumPy PCG64 ``default_rng``):

* ``small`` -- one 1024x1024 matrix, W ~ N(0, 0.05) from seed 0. This is the
  same call as the per-row int8/int4 worked example on the "ai-serving-optimise"
  page (section 2, "quantization: a scale and rounding"). Formats: int8 with
  one scale per row (g = 1024) and int4 with g = 32. x ~ N(0, 1) from seed 1.
* ``mid`` -- one 4096x4096 matrix, W ~ N(0, 0.02) from seed 2, with 0.1 % of
  the entries (16,777 distinct positions drawn without replacement) replaced
  by z * 20 * 0.02, z ~ N(0, 1). Formats: int4 g = 128 and int8 g = 128.
  x from seed 3 at M in {1, 8}.
* ``llama7b`` -- 32 decoder layers x {q, k, v, o: 4096x4096; gate, up:
  11008x4096; down: 4096x11008}, W ~ N(0, 0.02), seed 100 + 7*layer + index.
  Formats: int4 g = 128 and int8 with one scale per output channel (g = K).
  x from seed 4 (K = 4096) or 5 (K = 11008) at M in {1, 4, 16}.
* ``mlp70b`` -- gate/up 28672x8192 and down 8192x28672, W ~ N(0, 0.015) from
  seeds 6/7/8, 0.05 % outliers z * 20 * 0.015. Format int4 g = 64. x from
  seed 9 at M = 1.
* ``prefill`` -- x [2048, 4096] ~ N(0, 1) rounded to bfloat16 (round to
  nearest even), seed 10; W [14336, 4096] ~ N(0, 0.02), seed 11. Formats:
  int4 g = 128 and int8 per output channel.

The outliers stand in for the few large weights that the "Huit bits, puis
quatre" page (section on LLM.int8() outliers) describes as 3 to 20 times the
rest; no dataset or trained checkpoint is involved anywhere.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

__all__ = [
    "Matrix",
    "Workload",
    "WORKLOADS",
    "weight",
    "activations",
    "activations_bf16",
    "adversarial_rows",
]


@dataclass(frozen=True)
class Matrix:
    name: str
    N: int
    K: int
    sigma: float
    seed: int
    outlier_frac: float = 0.0

    @property
    def n_outliers(self) -> int:
        return int(self.N * self.K * self.outlier_frac)


@dataclass(frozen=True)
class Workload:
    name: str
    matrices: Tuple[Matrix, ...]
    formats: Tuple[Tuple[int, Optional[int]], ...]  # (bits, group); None = per output channel (g = K)
    Ms: Tuple[int, ...]
    x_seeds: Tuple[Tuple[int, int], ...]  # (K, seed)
    x_dtype: str = "f32"
    description: str = ""

    def x_seed(self, K: int) -> int:
        for k, s in self.x_seeds:
            if k == K:
                return s
        raise KeyError(K)

    def group(self, fmt_index: int, K: int) -> int:
        bits, g = self.formats[fmt_index]
        return K if g is None else g


def _llama_mats() -> Tuple[Matrix, ...]:
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    out = []
    for layer in range(32):
        for idx, (nm, n, k) in enumerate(shapes):
            out.append(Matrix(f"L{layer}.{nm}", n, k, 0.02, 100 + 7 * layer + idx))
    return tuple(out)


WORKLOADS = {
    "small": Workload(
        "small",
        (Matrix("W", 1024, 1024, 0.05, 0),),
        ((8, 1024), (4, 32)),
        (1,),
        ((1024, 1),),
        description="1024x1024 W~N(0,0.05) seed 0; int8 per-row (g=1024), int4 g=32; M=1",
    ),
    "mid": Workload(
        "mid",
        (Matrix("W", 4096, 4096, 0.02, 2, 0.001),),
        ((4, 128), (8, 128)),
        (1, 8),
        ((4096, 3),),
        description="4096x4096 W~N(0,0.02)+0.1% 20x outliers; int4 g=128, int8 g=128; M in {1,8}",
    ),
    "llama7b": Workload(
        "llama7b",
        _llama_mats(),
        ((4, 128), (8, None)),
        (1, 4, 16),
        ((4096, 4), (11008, 5)),
        description="Llama-7B decoder linear stack, 32 layers x {q,k,v,o,gate,up,down}; int4 g=128, int8 per-channel",
    ),
    "mlp70b": Workload(
        "mlp70b",
        (Matrix("gate", 28672, 8192, 0.015, 6, 0.0005),
         Matrix("up", 28672, 8192, 0.015, 7, 0.0005),
         Matrix("down", 8192, 28672, 0.015, 8, 0.0005)),
        ((4, 64),),
        (1,),
        ((8192, 9), (28672, 9)),
        description="70B-shaped MLP (gate/up 28672x8192, down 8192x28672), 0.05% 20x outliers; int4 g=64; M=1",
    ),
    "prefill": Workload(
        "prefill",
        (Matrix("W", 14336, 4096, 0.02, 11),),
        ((4, 128), (8, None)),
        (2048,),
        ((4096, 10),),
        x_dtype="bf16",
        description="prefill M=2048, K=4096, N=14336, x~N(0,1) bf16; int4 g=128, int8 per-channel",
    ),
}


def weight(m: Matrix) -> np.ndarray:
    """W[N, K] fp32 for one matrix spec: N(0, sigma) then optional outliers."""
    rng = np.random.default_rng(m.seed)
    w = rng.normal(0.0, m.sigma, (m.N, m.K)).astype(np.float32)
    n_out = m.n_outliers
    if n_out:
        pos = rng.choice(m.N * m.K, n_out, replace=False)
        z = rng.normal(0.0, 1.0, n_out)
        w.reshape(-1)[pos] = (z * 20.0 * m.sigma).astype(np.float32)
    return w


def activations(M: int, K: int, seed: int) -> np.ndarray:
    """x[M, K] fp32 ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    return rng.normal(0.0, 1.0, (M, K)).astype(np.float32)


def activations_bf16(M: int, K: int, seed: int):
    """x[M, K] as a CPU torch.bfloat16 tensor (fp32 draws rounded to nearest even).

    Widening the result back with ``.float()`` is exact, so the oracle sees
    exactly the values the GPU receives.
    """
    import torch

    return torch.from_numpy(activations(M, K, seed)).to(torch.bfloat16)


def adversarial_rows(K: int, seed: int = 1234) -> np.ndarray:
    """Rows built to stress the rounding/packing edge cases (K a multiple of 16).

    Row kinds, in order:
      0 all zeros;
      1 a single nonzero;
      2 int4 ties: every 16th entry is 7 * 2^-4 and the rest are (k + 1/2) * 2^-4
        with k in [-7, 6], so any group of 16 aligned entries has a power-of-two
        int4 step 2^-4 and w / step lands exactly on half-integers;
      3 int8 ties: the same with 127 * 2^-8 and (k + 1/2) * 2^-8, k in [-127, 126];
      4 fp32 subnormals;
      5 a step that underflows to zero: entries in {0, +-2^-149};
      6 +absmax and -absmax both present;
      7 one repeated negative value;
      8 one huge value among tiny ones;
      9 random normals.
    """
    rng = np.random.default_rng(seed)
    rows: List[np.ndarray] = []
    rows.append(np.zeros(K, np.float32))
    r = np.zeros(K, np.float32); r[K // 3] = -0.75; rows.append(r)
    t4 = (rng.integers(-7, 7, K).astype(np.float64) + 0.5) * 2.0 ** -4
    t4[::16] = 7 * 2.0 ** -4
    rows.append(t4.astype(np.float32))
    t8 = (rng.integers(-127, 127, K).astype(np.float64) + 0.5) * 2.0 ** -8
    t8[::16] = 127 * 2.0 ** -8
    rows.append(t8.astype(np.float32))
    rows.append((rng.normal(0, 1, K) * 1e-40).astype(np.float32))
    tiny = np.float32(2.0 ** -149)
    rows.append((rng.integers(-1, 2, K) * tiny).astype(np.float32))
    r = rng.normal(0, 0.1, K).astype(np.float32); r[1] = 2.0; r[K - 2] = -2.0; rows.append(r)
    rows.append(np.full(K, -0.3, np.float32))
    r = (rng.normal(0, 1, K) * 1e-6).astype(np.float32); r[5] = 3.0e4; rows.append(r)
    rows.append(rng.normal(0, 1, K).astype(np.float32))
    return np.stack(rows)
