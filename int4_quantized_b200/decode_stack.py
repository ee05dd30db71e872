"""Decode through a whole Llama-7B-shaped linear stack: 32 layers x {q, k, v, o: 4096x4096;
gate, up: 11008x4096; down: 4096x11008}, i.e. 224 quantized GEMVs per token step.

    python -m int4_quantized_b200.decode_stack [--bits 4] [--group 128] [--reps 20]

Weights: W ~ N(0, 0.02) drawn on the device (one seeded generator per matrix, seed
100 + 7 * layer + index; the timing does not depend on the values) and packed with qpack.
The matrices that read the same activations are packed into one contiguous buffer per
layer (q|k|v and gate|up): groups run along K, so the payload of the stacked matrix is
byte for byte the three (or two) payloads one after the other, and one GEMV of 12288 (or
22016) rows covers them.

One token step has data flow: level 0 of a layer reads the layer input h and writes
q|k|v; o reads q (the attention is not part of this path); gate|up read o's output; down
reads gate (the activation function is not part of this path) and its output is the next
layer's h. Three ways to run the step are timed:
  persistent  one launch of the decode-stack kernel (q4_stack_run) for all 224 GEMVs
  graph       the 128 qgemm calls of the fused matrices, captured in one CUDA graph, each
              call declaring its weights static (launch overlap)
  graph_224   the 224 separate qgemm calls, likewise
The stack (3.4 GB packed at int4 g128, 6.5 GB at int8 per channel) is far larger than L2,
so every step reads the weights from HBM. Reported: microseconds per step and GB/s of
packed weights + scales.
"""
from __future__ import annotations

import argparse
import json
from typing import Dict, List, Optional

import torch

from . import DecodeStack, StackGemv, qgemm, qgemm_workspace_bytes, qpack

D, F = 4096, 11008
SHAPES = (("q", D, D), ("k", D, D), ("v", D, D), ("o", D, D), ("gate", F, D), ("up", F, D), ("down", D, F))
# matrices packed back to back (they read the same x): one fused GEMV each
FUSED = (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")), ("down", ("down",)))
LEVEL = {"qkv": 0, "o": 1, "gate_up": 2, "down": 3}


class Matrix:
    """One matrix of the stack: views of its payload and scales inside the fused buffers."""

    def __init__(self, name, layer, N, K, group, payload, scales):
        self.name, self.layer, self.N, self.K, self.group = name, layer, N, K, group
        self.payload, self.scales = payload, scales


class Fused:
    """A fused GEMV: the matrices `parts`, back to back."""

    def __init__(self, name, layer, parts: List[Matrix], payload, scales):
        self.name, self.layer, self.parts = name, layer, parts
        self.N = sum(m.N for m in parts)
        self.K = parts[0].K
        self.group = parts[0].group
        self.payload, self.scales = payload, scales


def build_stack(bits: int, group: Optional[int], layers: int = 32, device=None, sigma: float = 0.02):
    """[Fused] of every layer (q|k|v, o, gate|up, down), weights packed in place."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    shapes = {n: (N, K) for n, N, K in SHAPES}
    idx = {n: i for i, (n, _, _) in enumerate(SHAPES)}
    out = []
    for layer in range(layers):
        for fname, parts in FUSED:
            K = shapes[parts[0]][1]
            g = K if group is None else group
            Ns = [shapes[p][0] for p in parts]
            payload = torch.empty(sum(Ns) * K * bits // 8, dtype=torch.uint8, device=dev)
            scales = torch.empty(sum(Ns) * K // g, dtype=torch.float32, device=dev)
            mats, r0 = [], 0
            for p, N in zip(parts, Ns):
                gen = torch.Generator(device=dev).manual_seed(100 + 7 * layer + idx[p])
                w = torch.randn(N, K, device=dev, generator=gen) * sigma
                pv = payload[r0 * K * bits // 8:(r0 + N) * K * bits // 8]
                sv = scales[r0 * K // g:(r0 + N) * K // g]
                qpack(w, bits, g, payload=pv, scales=sv)
                del w
                mats.append(Matrix(p, layer, N, K, g, pv, sv))
                r0 += N
            out.append(Fused(fname, layer, mats, payload, scales))
    return out


def stack_bytes(stack) -> int:
    return sum(f.payload.numel() + 4 * f.scales.numel() for f in stack)


class Activations:
    """The step's activation buffers with the data flow of the module docstring."""

    def __init__(self, stack, x_dtype=torch.float32, seed: int = 4):
        dev = stack[0].payload.device
        layers = max(f.layer for f in stack) + 1
        gen = torch.Generator(device=dev).manual_seed(seed)
        self.h0 = torch.randn(D, device=dev, generator=gen).to(x_dtype)
        self.y: Dict[tuple, torch.Tensor] = {}
        for f in stack:
            self.y[(f.layer, f.name)] = torch.empty(f.N, dtype=torch.float32, device=dev)
        self.x_dtype = x_dtype
        self.layers = layers

    def x_of(self, f: Fused) -> torch.Tensor:
        if self.x_dtype != torch.float32:
            return self.h0  # bf16 activations: every GEMV reads the (bf16) step input
        if f.name == "qkv":
            return self.h0 if f.layer == 0 else self.y[(f.layer - 1, "down")]
        if f.name == "o":
            return self.y[(f.layer, "qkv")][:D]  # q
        if f.name == "gate_up":
            return self.y[(f.layer, "o")]
        return self.y[(f.layer, "gate_up")][:F]  # gate

    def y_of(self, f: Fused, part: Optional[Matrix] = None) -> torch.Tensor:
        y = self.y[(f.layer, f.name)]
        if part is None:
            return y
        r0 = 0
        for m in f.parts:
            if m is part:
                return y[r0:r0 + m.N]
            r0 += m.N
        raise KeyError(part.name)


def make_decode_stack(stack, bits: int, x_dtype=torch.float32, fused: bool = False):
    """The persistent decode stack of the step (fused=False: the 224 matrices as GEMVs)."""
    acts = Activations(stack, x_dtype)
    gemvs = []
    for f in stack:
        lvl = 4 * f.layer + LEVEL[f.name]
        x = acts.x_of(f)
        if fused:
            gemvs.append(StackGemv(f.payload, f.scales, x, acts.y_of(f), f.N, f.K, f.group, lvl))
        else:
            for m in f.parts:
                gemvs.append(StackGemv(m.payload, m.scales, x, acts.y_of(f, m), m.N, m.K, m.group, lvl))
    return DecodeStack(gemvs, bits), acts


def _time(fn, reps: int, warmup: int, stream) -> float:
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def time_persistent(stack, bits: int, reps: int = 20, warmup: int = 3, fused: bool = False) -> dict:
    """One launch of the decode-stack kernel per step."""
    dstack, _ = make_decode_stack(stack, bits, fused=fused)
    stream = torch.cuda.Stream(device=stack[0].payload.device)
    status = torch.zeros(1, dtype=torch.int32, device=stack[0].payload.device)
    us = _time(lambda: dstack.run(status), reps, warmup, stream)
    assert int(status.item()) == 0, "a bounded wait in the decode-stack kernel gave up"
    nbytes = stack_bytes(stack)
    return {"mode": "persistent", "M": 1, "us_per_step": round(us, 1), "gemvs": len(dstack.gemvs), "launches": 1,
            "weight_bytes": nbytes, "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)}


def capture_step(stack, bits: int, acts: Optional[Activations] = None, M: int = 1, weights_static: bool = True,
                 fused: bool = True):
    """The step's qgemm calls captured in one CUDA graph (M rows of x per call).

    M = 1 keeps the data flow through `acts`; M > 1 reads fixed activations (one [M, K]
    buffer per K). Returns (graph, stream, number of calls, buffers to keep alive)."""
    dev = stack[0].payload.device
    calls = []
    if M == 1:
        acts = acts or Activations(stack)
        for f in stack:
            x = acts.x_of(f).reshape(1, -1)
            if fused:
                calls.append((x, f.payload, f.scales, f.N, f.K, f.group, acts.y_of(f).reshape(1, -1)))
            else:
                for m in f.parts:
                    calls.append((x, m.payload, m.scales, m.N, m.K, m.group, acts.y_of(f, m).reshape(1, -1)))
    else:
        gen = torch.Generator(device=dev).manual_seed(4)
        xs = {K: torch.randn(M, K, device=dev, generator=gen) for K in (D, F)}
        for f in stack:
            parts = [f] if fused else f.parts
            for m in parts:
                calls.append((xs[m.K], m.payload, m.scales, m.N, m.K, m.group,
                              torch.empty(M, m.N, device=dev)))
    ws = {}
    for x, p, s, N, K, g, y in calls:
        nb = qgemm_workspace_bytes(M, N, K, bits, g)
        if nb and (N, K) not in ws:
            ws[(N, K)] = torch.empty(nb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        for x, p, s, N, K, g, y in calls:
            qgemm(x, p, s, N, K, bits, g, out=y, workspace=ws.get((N, K)), weights_static=weights_static)

    with torch.cuda.stream(stream):
        step()  # every code path once outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    return graph, stream, len(calls), (calls, ws, acts)


def time_graph(stack, bits: int, M: int = 1, reps: int = 20, warmup: int = 3, weights_static: bool = True,
               fused: bool = True) -> dict:
    """capture_step, replayed: microseconds per step."""
    graph, stream, ncalls, keep = capture_step(stack, bits, None, M, weights_static, fused)
    us = _time(graph.replay, reps, warmup, stream)
    del graph, keep
    nbytes = stack_bytes(stack)
    return {"mode": "graph" if fused else "graph_224", "M": M, "us_per_step": round(us, 1), "gemvs": ncalls,
            "weight_bytes": nbytes, "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1), "weights_static": weights_static}


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8])
    ap.add_argument("--group", type=int, default=128, help="0 = one scale per output channel")
    ap.add_argument("--M", type=int, nargs="+", default=[1])
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--layers", type=int, default=32)
    a = ap.parse_args()
    stack = build_stack(a.bits, a.group or None, a.layers)
    info = {"bits": a.bits, "group": a.group or "per-channel", "layers": a.layers}
    print(json.dumps({**time_persistent(stack, a.bits, a.reps), **info}), flush=True)
    for M in a.M:
        print(json.dumps({**time_graph(stack, a.bits, M, a.reps), **info}), flush=True)
        if M == 1:
            print(json.dumps({**time_graph(stack, a.bits, M, a.reps, fused=False), **info}), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
