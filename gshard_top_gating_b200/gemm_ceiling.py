"""The layer's expert GEMM stages against cuBLAS batched GEMMs of the same shapes.

    python -m gshard_top_gating_b200.gemm_ceiling --workload large --reps 30

A B200 under its 1 kW cap settles at an SM clock set by power, so a GEMM timed
alone on a cool GPU and one timed inside a long loop differ by 20% or more.  This
driver times both in the same power state: every repetition runs one layer
forward through the C ABI (moe_forward, with per-stage CUDA events) and then
torch.bmm over [E, C, M] x [E, M, H] and [E, C, H] x [E, H, M], the first and
second expert GEMMs with every expert at capacity C.  cuBLAS is the library
baseline here; the layer never calls it.

Both GEMMs are reported in ms and TFLOP/s.  The layer's useful work is
2*A*M*H per GEMM (A kept assignments); its tiles cover ceil(n_e / tile rows)
row tiles per expert, which at capacity is the E*C rows the batched GEMM does.
Prints one JSON line.  Needs a GPU.
"""
from __future__ import annotations

import argparse
import json
import statistics
import time

import torch

from . import _lib as L
from .inputs import WORKLOADS, make_inputs
from .layer import MoeLayer


def _clock_sampler():
    try:
        import bench                      # the repository's bench.py, when run from the repo root
        return bench.ClockSampler(torch.cuda.current_device()).__enter__()
    except Exception:
        return None


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", choices=[n for n, w in WORKLOADS.items() if w.act == "bf16"],
                    default="large")
    ap.add_argument("--reps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    x, Wg, b, W1, W2 = make_inputs(w, device=dev)
    layer = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y = torch.empty_like(x)
    C = layer.capacity(w.S)
    E, M, H = w.E, w.M, w.H
    xe = torch.randn(E, C, M, device=dev, dtype=torch.bfloat16)
    he = torch.empty(E, C, H, device=dev, dtype=torch.bfloat16)
    ye = torch.empty(E, C, M, device=dev, dtype=torch.bfloat16)
    W1v, W2v = W1.view(E, M, H), W2.view(E, H, M)

    for _ in range(args.warmup):
        layer(x, out=y)
        torch.bmm(xe, W1v, out=he)
        torch.bmm(he, W2v, out=ye)
    torch.cuda.synchronize()
    _, _, _, cnt = layer.routing(w.S)
    A = int(torch.clamp(cnt.long(), max=C).sum().item())

    L.moe_set_profiling(layer.h, True)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.reps)]
    stages = []
    clk = _clock_sampler()
    t0 = time.monotonic()
    for r in range(args.reps):
        layer(x, out=y)
        stages.append(L.moe_get_stage_times(layer.h))
        ev[r][0].record()
        torch.bmm(xe, W1v, out=he)
        ev[r][1].record()
        torch.bmm(he, W2v, out=ye)
        ev[r][2].record()
    torch.cuda.synchronize()
    t1 = time.monotonic()
    L.moe_set_profiling(layer.h, False)
    clocks = clk.summary(t0, t1, "interleaved loop") if clk else None
    if clk:
        clk.__exit__(None, None, None)

    med = statistics.median
    ffn1 = med(s[L.STAGES.index("ffn1")] for s in stages)
    ffn2 = med(s[L.STAGES.index("ffn2")] for s in stages)
    bmm1 = med(e[0].elapsed_time(e[1]) for e in ev)
    bmm2 = med(e[1].elapsed_time(e[2]) for e in ev)
    useful = 2.0 * A * M * H
    full = 2.0 * E * C * M * H
    tf = lambda flop, ms: round(flop / (ms * 1e-3) / 1e12, 1)
    print(json.dumps({
        "workload": args.workload, "reps": args.reps, "A": A, "E_times_C": E * C,
        "layer_ms": {"ffn1": round(ffn1, 4), "ffn2": round(ffn2, 4)},
        "layer_tflops_useful": {"ffn1": tf(useful, ffn1), "ffn2": tf(useful, ffn2)},
        "cublas_bmm_ms": {"ffn1": round(bmm1, 4), "ffn2": round(bmm2, 4)},
        "cublas_bmm_tflops": {"ffn1": tf(full, bmm1), "ffn2": tf(full, bmm2)},
        "clocks": clocks,
    }))
    layer.close()


if __name__ == "__main__":
    main()
