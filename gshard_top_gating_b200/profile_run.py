"""Run a few layer forwards of one workload, for a profiler such as ncu.

    python -m gshard_top_gating_b200.profile_run --workload large --forwards 4
    python -m gshard_top_gating_b200.profile_run --workload large --hidden 64   # narrow experts
    python -m gshard_top_gating_b200.profile_run --workload large --tokens 16384 --experts 16

The token batch, gate and expert count are the workload's unless replaced:
--hidden replaces the expert width H, so the router, capacity scan, dispatch and
combine run on the full batch while the expert weights (and the device memory a
profiler saves and restores between its passes) stay small; --tokens and
--experts replace S and E together, which keeps the per-expert GEMM shapes
(capacity k*S/E rows, M x H weights) with fewer experts.  Every forward goes
through the C ABI (moe_forward); nothing is timed here.
"""
from __future__ import annotations

import argparse

import torch

from .inputs import WORKLOADS, make_inputs
from .layer import MoeLayer


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", choices=list(WORKLOADS), default="large")
    ap.add_argument("--forwards", type=int, default=4)
    ap.add_argument("--hidden", type=int, default=0, help="expert width H to use instead of the workload's")
    ap.add_argument("--tokens", type=int, default=0, help="token count S to use instead of the workload's")
    ap.add_argument("--experts", type=int, default=0, help="expert count E to use instead of the workload's")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.hidden:
        w = w.with_(H=args.hidden)
    if args.tokens:
        w = w.with_(S=args.tokens)
    if args.experts:
        w = w.with_(E=args.experts)
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    layer = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y = torch.empty_like(x)
    for _ in range(args.forwards):
        layer(x, out=y)
    torch.cuda.synchronize()
    layer.close()
    print(f"profile_run: {args.forwards} forwards of {w.name} (S={w.S}, M={w.M}, H={w.H}, E={w.E}, k={w.k})")


if __name__ == "__main__":
    main()
