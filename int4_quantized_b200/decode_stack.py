"""Decode through a whole Llama-7B-shaped linear stack: 32 layers x {q, k, v, o: 4096x4096;
gate, up: 11008x4096; down: 4096x11008}, i.e. 224 quantized GEMVs per token step.

    python -m int4_quantized_b200.decode_stack [--bits 4] [--group 128] [--M 1 4 16] [--reps 20]

The weights are drawn on the device (N(0, 0.02), one seeded generator per matrix, seed
100 + 7 * layer + index) and packed with qpack; x ~ N(0, 1). One token step is the 224
qgemm calls in layer order, captured once in a CUDA graph (launch overhead is what
dominates a stack of small GEMVs), and replayed. The stack (3.4 GB packed at int4 g128,
6.5 GB at int8 per channel) is far larger than L2, so every step reads the weights from
HBM. Reported: microseconds per token step and the GB/s of packed weights + scales.

With --static (the default) every call declares its weights static
(Q4_QGEMM_WEIGHTS_STATIC): each GEMV streams its weights while the one before it
finishes, as they are packed once and never written during the step; --plain times the
same step with strict stream order.
"""
from __future__ import annotations

import argparse
import json
from typing import List, Optional, Tuple

import torch

from . import qgemm, qgemm_workspace_bytes, qpack

SHAPES = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
          ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))


def build_stack(bits: int, group: Optional[int], layers: int = 32, device=None) -> List[Tuple]:
    """[(N, K, group, payload, scales)] for every matrix of the stack, in layer order."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    stack = []
    for layer in range(layers):
        for idx, (_, N, K) in enumerate(SHAPES):
            gen = torch.Generator(device=dev).manual_seed(100 + 7 * layer + idx)
            w = torch.randn(N, K, device=dev, generator=gen) * 0.02
            g = K if group is None else group
            payload, scales = qpack(w, bits, g)
            del w
            stack.append((N, K, g, payload, scales))
    return stack


def stack_bytes(stack) -> int:
    return sum(p.numel() + 4 * s.numel() for _, _, _, p, s in stack)


def time_stack(stack, bits: int, M: int, reps: int = 20, warmup: int = 3, weights_static: bool = True) -> dict:
    """Capture the token step (all GEMVs of the stack) in a CUDA graph and time it."""
    dev = stack[0][3].device
    gen = torch.Generator(device=dev).manual_seed(4)
    xs = {K: torch.randn(M, K, device=dev, generator=gen) for K in sorted({k for _, k, _, _, _ in stack})}
    ys = {N: torch.empty(M, N, device=dev) for N in sorted({n for n, _, _, _, _ in stack})}
    ws = {}
    for N, K, g, _, _ in stack:
        nb = qgemm_workspace_bytes(M, N, K, bits, g)
        if nb and (N, K, g) not in ws:
            ws[(N, K, g)] = torch.empty(nb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        for N, K, g, p, s in stack:
            qgemm(xs[K], p, s, N, K, bits, g, out=ys[N], workspace=ws.get((N, K, g)),
                  weights_static=weights_static)

    with torch.cuda.stream(stream):
        step()  # every code path once outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = stack_bytes(stack)
    del graph
    return {"M": M, "us_per_step": round(us, 1), "gemvs": len(stack), "weight_bytes": nbytes,
            "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1), "weights_static": weights_static}


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8])
    ap.add_argument("--group", type=int, default=128, help="0 = one scale per output channel")
    ap.add_argument("--M", type=int, nargs="+", default=[1, 4, 16])
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--plain", action="store_true", help="strict stream order (no static-weights flag)")
    ap.add_argument("--both", action="store_true", help="time both modes")
    a = ap.parse_args()
    stack = build_stack(a.bits, a.group or None, a.layers)
    modes = (False, True) if a.both else (not a.plain,)
    for M in a.M:
        for static in modes:
            r = time_stack(stack, a.bits, M, a.reps, weights_static=static)
            r.update(bits=a.bits, group=a.group or "per-channel", layers=a.layers)
            print(json.dumps(r), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
