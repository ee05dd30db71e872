"""Run one library call on a seeded synthetic shape and time it (CUDA events).

    python -m int4_quantized_b200.run_case qgemm N K bits group M [--bf16] [--reps R]
    python -m int4_quantized_b200.run_case qpack N K bits group [--reps R]

W ~ N(0, 0.02) and x ~ N(0, 1) are drawn on the device from a fixed seed. The call is
made `--warmup` times untimed, then `--reps` times with a CUDA event pair around each; the
median and the achieved rates are printed as one JSON line (GB/s of the algorithmic bytes:
payload + scales for qgemm, fp32 input + payload + scales for qpack; TFLOP/s for qgemm).
The same command line is what a profiler is pointed at to capture a single kernel.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import qgemm, qpack


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("kind", choices=["qgemm", "qpack"])
    ap.add_argument("N", type=int)
    ap.add_argument("K", type=int)
    ap.add_argument("bits", type=int, choices=[4, 8])
    ap.add_argument("group", type=int)
    ap.add_argument("M", type=int, nargs="?", default=1)
    ap.add_argument("--bf16", action="store_true", help="x in bfloat16 (qgemm)")
    ap.add_argument("--reps", type=int, default=10)
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
        call = lambda: qgemm(x, payload, scales, a.N, a.K, a.bits, a.group, out=y)  # noqa: E731
        nbytes = pbytes
    else:
        call = lambda: qpack(w, a.bits, a.group, payload=payload, scales=scales)  # noqa: E731
        nbytes = 4 * w.numel() + pbytes
    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(a.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    us = statistics.median(times)
    out = {"kind": a.kind, "N": a.N, "K": a.K, "bits": a.bits, "group": a.group, "us_median": round(us, 3),
           "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)}
    if a.kind == "qgemm":
        out.update(M=a.M, x="bf16" if a.bf16 else "f32", TFLOPs=round(2.0 * a.M * a.N * a.K / (us * 1e-6) / 1e12, 2))
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
