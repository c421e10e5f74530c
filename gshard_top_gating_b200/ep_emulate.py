"""Expert-parallel forward of one workload, G ranks emulated on one GPU, timed per rank.

    python -m gshard_top_gating_b200.ep_emulate --workload large --ranks 8 --phases 2
    python -m gshard_top_gating_b200.ep_emulate --workload large --ranks 8 --peers --check

Each rank is its own library handle with S/G tokens and E/G experts, as in
`ep.ep_forward_local`.  The ranks run one after another on one device, so each
rank's kernels are timed alone with CUDA events: route (router and per-rank scan),
dispatch (plan upload and pack), the experts of each phase (unpack, both grouped
GEMMs, repack) and combine.  The exchanges between ranks are device copies here and
are not timed; the JSON line reports the rows and bytes each rank would send and
receive per phase, from which a transport's time follows.  With --peers the pack
writes into the owners' receive buffers and the combine reads from them (every buffer
on the one device stands in for a peer's).  --check compares the concatenated output
with the one-device layer's on the whole batch, bit for bit.  Needs a GPU.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from .ep import EPMoeLayer, _exchange
from .inputs import WORKLOADS, make_inputs
from .layer import MoeLayer


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", choices=[n for n, w in WORKLOADS.items() if w.act == "bf16"],
                    default="large")
    ap.add_argument("--ranks", type=int, default=8)
    ap.add_argument("--phases", type=int, choices=(1, 2), default=2)
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--peers", action="store_true", help="pack and combine over peer memory (one phase)")
    ap.add_argument("--check", action="store_true", help="compare with the one-device layer, bit for bit")
    args = ap.parse_args()
    if args.peers:
        args.phases = 1
    w = WORKLOADS[args.workload]
    G = args.ranks
    if w.E % G or w.S % G:
        raise SystemExit("the workload's E and S must divide by --ranks")
    dev = torch.device("cuda", torch.cuda.current_device())
    x, Wg, b, W1, W2 = make_inputs(w, device=dev)
    El, Sg = w.E // G, w.S // G
    layers = [EPMoeLayer(G, g, Sg, w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b,
                         W1[g * El:(g + 1) * El].contiguous(), W2[g * El:(g + 1) * El].contiguous(),
                         phases=args.phases) for g in range(G)]
    xs = [x[g * Sg:(g + 1) * Sg].contiguous() for g in range(G)]
    ys = [torch.empty_like(xg) for xg in xs]
    if args.peers:
        ptrs = [layer.recvbuf.data_ptr() for layer in layers]
        for layer in layers:
            layer.set_peers(ptrs)

    def timed(fn):
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        z.record()
        return a, z

    stages = ["route", "dispatch"] + [f"experts_phase{p}" for p in range(args.phases)] + ["combine"]
    times = {s: [[] for _ in range(G)] for s in stages}
    for rep in range(args.reps + 1):               # the first pass warms up
        ev = {s: [None] * G for s in stages}
        for g, layer in enumerate(layers):
            ev["route"][g] = timed(lambda: layer.route(xs[g]))
        stats_all = torch.stack([layer.stats for layer in layers]).cpu().numpy()
        if args.peers:
            for g, layer in enumerate(layers):
                ev["dispatch"][g] = timed(lambda: layer.dispatch_to_peers(stats_all, xs[g]))
            for g, layer in enumerate(layers):
                ev["experts_phase0"][g] = timed(lambda: layer.experts())
            for g, layer in enumerate(layers):
                ev["combine"][g] = timed(lambda: layer.combine_from_peers(ys[g]))
        else:
            for g, layer in enumerate(layers):
                ev["dispatch"][g] = timed(lambda: layer.dispatch(stats_all, xs[g]))
            for p in range(args.phases):
                _exchange(layers, p)
                for g, layer in enumerate(layers):
                    ev[f"experts_phase{p}"][g] = timed(lambda: layer.experts_phase(p))
                _exchange(layers, p, back=True)
            for g, layer in enumerate(layers):
                ev["combine"][g] = timed(lambda: layer.combine(ys[g]))
        torch.cuda.synchronize()
        if rep:
            for s in stages:
                for g in range(G):
                    times[s][g].append(ev[s][g][0].elapsed_time(ev[s][g][1]))
    med = {s: [statistics.median(v) for v in times[s]] for s in stages}
    row_bytes = w.M * 2
    per_rank = []
    for g, layer in enumerate(layers):
        sr, rr = layer.send_rows, layer.recv_rows
        per_rank.append({
            "rank": g, "ms": {s: round(med[s][g], 4) for s in stages},
            "send_rows_per_phase": [int(v) for v in sr.sum(axis=1)],
            "recv_rows_per_phase": [int(v) for v in rr.sum(axis=1)],
            "remote_send_MB_per_phase": [round((int(sr[p].sum()) - int(sr[p][g])) * row_bytes / 1e6, 2)
                                         for p in range(args.phases)],
            "remote_recv_MB_per_phase": [round((int(rr[p].sum()) - int(rr[p][g])) * row_bytes / 1e6, 2)
                                         for p in range(args.phases)],
        })
    compute = {s: round(max(med[s]), 4) for s in stages}
    check = None
    if args.check:
        one = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
        y1 = one(x)
        torch.cuda.synchronize()
        y = torch.cat(ys)
        check = {"bitwise_equal_to_one_device": bool(torch.equal(y, y1)),
                 "max_abs_diff": float((y.float() - y1.float()).abs().max())}
        one.close()
    print(json.dumps({
        "workload": f"{w.name} (S={w.S}, M={w.M}, H={w.H}, E={w.E}, k={w.k}, cf={w.cf})",
        "ranks": G, "phases": args.phases, "transport": "peer memory" if args.peers else "all-to-all",
        "tokens_per_rank": Sg, "experts_per_rank": El, "check": check,
        "slowest_rank_ms": compute, "slowest_rank_compute_ms": round(sum(compute.values()), 4),
        "per_rank": per_rank,
    }))
    for layer in layers:
        layer.close()


if __name__ == "__main__":
    main()
