"""Run one library call on a seeded synthetic shape and time it (CUDA events).

    python -m int4_quantized_b200.run_case qgemm N K bits group M [--bf16] [--static] [--reps R]
    python -m int4_quantized_b200.run_case qpack N K bits group [--reps R]

W ~ N(0, 0.02) and x ~ N(0, 1) are drawn on the device from a fixed seed. The inputs are
copied until the copies exceed twice the 126 MB L2 (at most 64 copies), and the calls
cycle through them, so that every call reads its weights from HBM. `--reps` calls are
captured in one CUDA graph (launched `--warmup` times untimed, then `--batches` times
between CUDA events): the per-call time is the batch time over `--reps`, back-to-back
device time without the host's launch cost. Printed as one JSON line: the median and the
90th percentile of the per-call time over the batches and the achieved rates (at the median) (GB/s of the algorithmic bytes: payload +
scales for qgemm, fp32 input + payload + scales for qpack; TFLOP/s for qgemm).
`--static` declares the weights static (Q4_QGEMM_WEIGHTS_STATIC), so each call may
stream its weights while the one before it ends.
The same command line is what a profiler is pointed at to capture a single kernel.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import qgemm, qgemm_workspace_bytes, qpack

L2_BYTES = 126 * 2 ** 20


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("kind", choices=["qgemm", "qpack"])
    ap.add_argument("N", type=int)
    ap.add_argument("K", type=int)
    ap.add_argument("bits", type=int, choices=[4, 8])
    ap.add_argument("group", type=int)
    ap.add_argument("M", type=int, nargs="?", default=1)
    ap.add_argument("--bf16", action="store_true", help="x in bfloat16 (qgemm)")
    ap.add_argument("--static", action="store_true", help="weights static (qgemm)")
    ap.add_argument("--reps", type=int, default=10, help="calls per timed graph")
    ap.add_argument("--batches", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()

    dev = torch.device("cuda", torch.cuda.current_device())
    gen = torch.Generator(device=dev).manual_seed(a.seed)
    w = torch.randn(a.N, a.K, device=dev, generator=gen) * 0.02
    payload, scales = qpack(w, a.bits, a.group)
    pbytes = payload.numel() + 4 * scales.numel()
    if a.kind == "qgemm":
        del w
        x = torch.randn(a.M, a.K, device=dev, generator=gen)
        if a.bf16:
            x = x.to(torch.bfloat16)
        y = torch.empty(a.M, a.N, device=dev)
        ncopy = max(1, min(64, -(-2 * L2_BYTES // pbytes)))
        P = [payload] + [payload.clone() for _ in range(ncopy - 1)]
        S = [scales] + [scales.clone() for _ in range(ncopy - 1)]
        need = qgemm_workspace_bytes(a.M, a.N, a.K, a.bits, a.group, x.dtype)
        ws = torch.empty(max(256, need), dtype=torch.uint8, device=dev)

        def call(i):
            j = i % ncopy
            qgemm(x, P[j], S[j], a.N, a.K, a.bits, a.group, out=y, workspace=ws, weights_static=a.static)

        nbytes = pbytes
    else:
        ncopy = max(1, min(64, -(-2 * L2_BYTES // (4 * w.numel() + pbytes))))
        W = [w] + [w.clone() for _ in range(ncopy - 1)]
        P = [payload] + [payload.clone() for _ in range(ncopy - 1)]
        S = [scales] + [scales.clone() for _ in range(ncopy - 1)]

        def call(i):
            j = i % ncopy
            qpack(W[j], a.bits, a.group, payload=P[j], scales=S[j])

        nbytes = 4 * w.numel() + pbytes
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(a.reps):  # every code path once outside capture
            call(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(a.reps):
            call(i)
    times = []
    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            graph.replay()
        for _ in range(a.batches):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3 / a.reps)
    torch.cuda.synchronize()
    del graph
    us = statistics.median(times)
    p90 = sorted(times)[min(len(times) - 1, int(round(0.9 * (len(times) - 1))))]
    out = {"kind": a.kind, "N": a.N, "K": a.K, "bits": a.bits, "group": a.group, "us_median": round(us, 3),
           "us_p90": round(p90, 3),
           "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1), "copies": ncopy, "calls_per_graph": a.reps}
    if a.kind == "qgemm":
        out.update(M=a.M, x="bf16" if a.bf16 else "f32", static=a.static,
                   TFLOPs=round(2.0 * a.M * a.N * a.K / (us * 1e-6) / 1e12, 2))
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
