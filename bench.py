"""Benchmark of the GShard MoE layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload mid]

A step is one whole layer forward (router, capacity scan, dispatch, two grouped
expert GEMMs, combine, losses) over one batch of synthetic tokens already
resident in HBM.  The default workload is the mid configuration (S=8192
tokens, M=1024, H=4096, E=32, top-2, capacity factor 2.0, bf16).  L2 is flushed
(a 256 MB write) before every timed step and each step is timed with CUDA
events on the launching stream; the sum over the K steps is the timed region.

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica of the layer on its own GPU and batch (the forward has no exchange on
one GPU); the slowest rank's time gives the job throughput ("scaling": "weak").

--impl reference times the CPU oracle (the plain float64 restatement of the
method) on a bounded token sample of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gshard_top_gating_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ("router", "scan", "dispatch", "ffn1", "ffn2", "combine")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples, each stamped with the host's monotonic clock."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.monotonic()
            while not self.rows and time.monotonic() - t0 < 10.0:
                time.sleep(0.05)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append((time.monotonic(), parts))

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def count(self, t0, t1):
        return sum(1 for t, _ in self.rows if t0 <= t <= t1)

    def summary(self, t0, t1, window):
        rows = [r for t, r in self.rows if t0 <= t <= t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "window": window}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [v for v in (num(r[1]) for r in rows) if v is not None]
        mx = [v for v in (num(r[2]) for r in rows) if v is not None]
        pw = [v for v in (num(r[3]) for r in rows) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows), "window": window}


def dist_setup(n):
    if n <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import torch.distributed as dist
    from datetime import timedelta
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(v: float, world: int) -> float:
    """Slowest rank's value (every rank calls this at the same point)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's timed region."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def source_hash(files) -> str:
    """Hash of the given files under the library's csrc/ (the kernel a counter was taken on)."""
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "gshard_top_gating_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(cs, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, while its sources are unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != source_hash(ent.get("sources", [])):
        return None
    return ent.get("dram_bytes_per_launch")


def algorithmic(w, A, n_active):
    """Algorithmic work per launch of each stage (A kept assignments, n_active experts
    with a kept row): ("hbm", bytes), or ("gemm", flops, bytes) for an expert GEMM,
    whose bytes are its operands read once (the active experts' weights) and its
    result written once."""
    s = 2 if w.act == "bf16" else 4
    S, M, H, E, k = w.S, w.M, w.H, w.E, w.k
    wts = n_active * M * H * s
    return {
        "router": ("hbm", S * M * s + 4 * M * E + S * E * 4 + S * k * 12),
        "scan": ("hbm", 0),
        "dispatch": ("hbm", (S + A) * M * s),
        "ffn1": ("gemm", 2.0 * A * M * H, A * M * s + wts + A * H * s),
        "ffn2": ("gemm", 2.0 * A * M * H, A * H * s + wts + A * M * s),
        "combine": ("hbm", (A + S) * M * s + S * k * 12),
    }


def algorithmic_bwd(w, A, n_active, pad_rows, nsplit):
    """Algorithmic work per launch of each backward stage, as algorithmic().  The
    weight gradients are written for every expert (zeros for the empty ones: the
    default, MOE_BWD_SKIP_EMPTY_EXPERTS off); dP reads one mask bit per element."""
    s = 2 if w.act == "bf16" else 4
    S, M, H, E, k = w.S, w.M, w.H, w.E, w.k
    wts, grads = n_active * M * H * s, E * M * H * s
    f = 2.0 * A * M * H
    return {
        "gate_bwd": ("hbm", S * M * s + 2 * A * M * s + 2 * S * E * 4 + S * k * 16 + E * 4),
        "pad_zero": ("hbm", pad_rows * (2 * M + H) * s),
        "dW2": ("gemm", f, A * H * s + A * M * s + grads),
        "dP": ("gemm", f, A * M * s + wts + A * H // 8 + A * H * s),
        "dW1": ("gemm", f, A * M * s + A * H * s + grads),
        "dX_e": ("gemm", f, A * H * s + wts + A * M * s),
        "dx": ("hbm", (A + S) * M * s + S * E * 4 + M * E * 4 + S * k * 8),
        "dWg": ("hbm", S * M * s + S * E * 4 + 2 * nsplit * (M + 1) * E * 4),
    }


def stage_roof(entry, seconds, pk):
    """(bound, achieved, peak, unit) of one stage.  An expert GEMM is bound by the slower
    of its flops at the bf16 tensor peak and its bytes at the HBM peak (a GEMM over few
    rows per expert streams weights faster than it can use the tensor cores)."""
    if entry[0] == "gemm":
        flops, nbytes = entry[1], entry[2]
        if flops / (pk["bf16_tflops"] * 1e12) >= nbytes / (pk["hbm_gbs"] * 1e9):
            return "tensor", flops / seconds / 1e12, pk["bf16_tflops"], "TFLOP/s"
        return "hbm", nbytes / seconds / 1e9, pk["hbm_gbs"], "GB/s"
    return "hbm", entry[1] / seconds / 1e9, pk["hbm_gbs"], "GB/s"


def stage_entry(entry, ms, pk):
    b_, ach, peak, unit = stage_roof(entry, ms / 1e3, pk)
    return {"ms": round(ms, 4), unit: round(ach, 1), "frac_of_peak": round(ach / peak, 4),
            "bound": b_}


def measure_copies(args, x, xh, yh, stream):
    """The e2e step's copies without the layer: its input host -> device, its output
    device -> host, each direction alone and both at once on two streams (pinned host
    buffers, the same bytes per step).  The slower of "both" and the device step bounds
    what the overlapped host-buffer pipeline can reach."""
    xd = torch.empty_like(x)
    yd = torch.empty_like(x)
    other = torch.cuda.Stream()
    reps = max(3, min(args.steps, 50))

    def run(h2d, d2h):
        for _ in range(2):                          # warm-up
            if h2d:
                xd.copy_(xh, non_blocking=True)
            if d2h:
                yh.copy_(yd, non_blocking=True)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        other.wait_stream(stream)
        for _ in range(reps):
            if h2d:
                xd.copy_(xh, non_blocking=True)
            if d2h:
                with torch.cuda.stream(other):
                    yh.copy_(yd, non_blocking=True)
        stream.wait_stream(other)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    nbytes = x.numel() * x.element_size()
    h2d, d2h, both = run(True, False), run(False, True), run(True, True)
    return {"h2d_ms": round(h2d, 4), "d2h_ms": round(d2h, 4), "both_ms": round(both, 4),
            "h2d_GBps": round(nbytes / h2d / 1e6, 1), "d2h_GBps": round(nbytes / d2h / 1e6, 1)}


def measure_backward(args, w, weights, x, y, flush, stream, pk, A, n_e):
    """One training step = moe_forward + moe_backward of the same tokens, device-timed.

    On a handle of its own, in training mode from its first forward (the backward
    enabled first), as a training loop would use the layer."""
    from gshard_top_gating_b200 import _lib as L
    from gshard_top_gating_b200.inputs import upstream_grad
    from gshard_top_gating_b200.layer import MoeLayer
    dev = x.device
    dy = upstream_grad(w, device=dev)
    layer = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, *weights)
    layer.enable_backward()
    dx = torch.empty_like(x)
    dWg = torch.empty(w.M, w.E, dtype=torch.float32, device=dev)
    dbias = torch.empty(w.E, dtype=torch.float32, device=dev) if w.skew_bias else None
    dW1 = torch.empty(w.E, w.M, w.H, dtype=x.dtype, device=dev)
    dW2 = torch.empty(w.E, w.H, w.M, dtype=x.dtype, device=dev)
    a_aux, a_z = 0.01, 0.001

    def bwd():
        L.moe_backward(layer.h, w.S, x, dy, a_aux, a_z, dx, dWg, dbias, dW1, dW2)

    for _ in range(3):
        layer(x, out=y)
        bwd()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 50))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    for i in range(n):
        flush.zero_()
        ev[i][0].record(stream)
        layer(x, out=y)
        ev[i][1].record(stream)
        bwd()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    bwd_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    L.moe_set_profiling(layer.h, True)
    per = [[] for _ in L.BWD_STAGES]
    for _ in range(min(n, 20)):
        flush.zero_()
        layer(x, out=y)
        bwd()
        for j, t in enumerate(L.moe_get_backward_stage_times(layer.h)):
            per[j].append(t)
    L.moe_set_profiling(layer.h, False)
    torch.cuda.synchronize()
    stage_ms = {nm: statistics.mean(v) for nm, v in zip(L.BWD_STAGES, per)}
    pad_rows = int(sum(((int(v) + 63) // 64) * 64 - int(v) for v in n_e.tolist()))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tiles = ((w.M + 64) // 64) * ((w.E + 63) // 64)
    nsplit = max(1, min((2 * sms + tiles - 1) // tiles, (w.S + 255) // 256))
    n_active = int((n_e > 0).sum().item())
    algo = algorithmic_bwd(w, A, n_active, pad_rows, nsplit)
    stages = {nm: stage_entry(algo[nm], stage_ms[nm], pk) for nm in L.BWD_STAGES if stage_ms[nm] > 0}
    dom = max(stage_ms, key=lambda k_: stage_ms[k_])
    b_, ach, peak, unit = stage_roof(algo[dom], stage_ms[dom] / 1e3, pk)
    ffn = sum(stage_ms[k_] for k_ in ("dW2", "dP", "dW1", "dX_e"))
    launches = n * (L.moe_kernels_per_forward(layer.h, w.S) + L.moe_kernels_per_backward(layer.h, w.S))
    layer.close()
    return {
        "what": "moe_forward + moe_backward of the same tokens (dL/dy given; a_aux=0.01, a_z=0.001)",
        "tokens_per_s": round(w.S / ((fwd_ms + bwd_ms) / 1e3), 1),
        "ms_fwd": round(fwd_ms, 4), "ms_bwd": round(bwd_ms, 4), "steps": n,
        "expert_gemm_TFLOP/s": round(4 * 2.0 * A * w.M * w.H / (ffn / 1e3) / 1e12, 1) if ffn > 0 else None,
        "roofline": {"bound": b_, "kernel": dom, "achieved": round(ach, 2), "peak": peak, "unit": unit,
                     "frac": round(ach / peak, 4),
                     "peak_source": "measured, burst" if b_ == "tensor" else "measured",
                     "frac_of_sustained": (round(ach / pk["bf16_tflops_sustained"], 4)
                                           if b_ == "tensor" and pk.get("bf16_tflops_sustained") else None)},
        "stages": stages,
        "gpu_launches": launches,
    }


def run_ours(args, rank, world, local):
    w = WORKLOADS[args.workload]
    from gshard_top_gating_b200 import _lib as L
    from gshard_top_gating_b200.layer import MoeLayer
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x, Wg, b, W1, W2 = make_inputs(w, device=dev)
    layer = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MB > L2

    for _ in range(args.warmup):
        layer(x, out=y)
    torch.cuda.synchronize()
    _, _, slot, cnt = layer.routing(w.S)
    C = layer.capacity(w.S)
    n_e = torch.clamp(cnt.long(), max=C)
    A = int(n_e.sum().item())
    n_active = int((n_e > 0).sum().item())

    # ---- the step: one layer forward, replayed from a CUDA graph of moe_forward
    # (its six kernels and their programmatic dependencies) unless --eager
    graph = None
    launch_note = "eager moe_forward"
    if not args.eager:
        try:
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                layer(x, out=y)
            torch.cuda.current_stream().wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                layer(x, out=y)
            torch.cuda.synchronize()
            launch_note = "CUDA graph of moe_forward"
        except Exception as exc:            # capture unsupported: time eager calls instead
            graph = None
            launch_note = f"eager moe_forward (graph capture failed: {type(exc).__name__})"
            torch.cuda.synchronize()

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer(x, out=y)

    for _ in range(2):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K forwards, L2 flushed before each, device time per step
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clk = ClockSampler(local).__enter__()
    barrier(world)
    torch.cuda.synchronize()
    t_begin = time.monotonic()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t_end = time.monotonic()
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.S, args.steps, total_ms, world)

    # ---- per-stage device times (events recorded by the library on the same stream)
    L.moe_set_profiling(layer.h, True)
    per_stage = [[] for _ in STAGES]
    for i in range(args.steps):
        flush.zero_()
        layer(x, out=y)
        for j, t in enumerate(L.moe_get_stage_times(layer.h)):
            per_stage[j].append(t)
    L.moe_set_profiling(layer.h, False)
    stage_ms = {n: statistics.mean(v) for n, v in zip(STAGES, per_stage)}

    # ---- end to end through the C ABI with host buffers (copies inside the timed region)
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(2):
        layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    barrier(world)
    e_s.record(stream)
    for _ in range(args.steps):
        layer.forward_host(xh, yh)
    e_e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), world)
    nbytes = x.numel() * x.element_size()
    copies = measure_copies(args, x, xh, yh, stream)

    # clocks: the timed region itself when it held enough samples, else a soak of
    # the same forward right after it (the timed region was too short to sample)
    if clk.count(t_begin, t_end) >= 3:
        clocks = clk.summary(t_begin, t_end, "timed region")
    else:
        s0 = time.monotonic()
        while time.monotonic() - s0 < 1.5:
            for _ in range(20):
                flush.zero_()
                step()
            torch.cuda.synchronize()
        clocks = clk.summary(s0, time.monotonic(),
                             "1.5 s soak of the same step right after the timed region")
    clk.__exit__()

    pk, pk_kind = peaks()
    algo = algorithmic(w, A, n_active)
    dom = max(stage_ms, key=lambda n: stage_ms[n])
    bound, achieved, peak, unit = stage_roof(algo[dom], stage_ms[dom] / 1e3, pk)
    roof = {"bound": bound, "kernel": dom, "achieved": round(achieved, 2), "peak": peak,
            "unit": unit, "frac": round(achieved / peak, 4), "traffic": ncu_traffic(dom, w.name),
            "peak_source": f"{pk_kind}, burst" if bound == "tensor" else pk_kind,
            "frac_of_sustained": (round(achieved / pk["bf16_tflops_sustained"], 4)
                                  if bound == "tensor" and pk.get("bf16_tflops_sustained") else None)}
    stages = {n: stage_entry(algo[n], stage_ms[n], pk) for n in STAGES if stage_ms[n] > 0}

    train = (None if args.no_backward
             else measure_backward(args, w, (Wg, b, W1, W2), x, y, flush, stream, pk, A, n_e))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_budget, x, Wg, b, W1, W2)

    line = {
        "metric": "MoE-layer tokens/sec on 1 B200; FFN % of bf16 TC peak; dispatch/combine HBM GB/s",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.act, "data": "synthetic",
        "config": {"workload": f"{w.name} (S={w.S}, M={w.M}, H={w.H}, E={w.E}, k={w.k}, cf={w.cf})",
                   "S": w.S, "M": w.M, "H": w.H, "E": w.E, "k": w.k, "capacity_factor": w.cf,
                   "C": C, "kept_assignments": A, "active_experts": n_active,
                   "l2": "flushed before every timed step (256 MB write)",
                   "launch": launch_note,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof, "stages": stages,
        "e2e": {"value": round(job_throughput(w.S, args.steps, e2e_ms, world), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                "ms_per_step": round(e2e_ms / args.steps, 4),
                "copies_alone": copies},
        "gpu_launches": args.steps * L.moe_kernels_per_forward(layer.h, w.S),
        "clocks": clocks,
        "cpu_baseline": cpu,
        "train_step": train,
    }
    layer.close()
    return line


def _oracle_inputs(w, x, Wg, b, W1, W2):
    """Host float64 copies of the workload's inputs (the oracle's input form)."""
    import numpy as np
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    return (f64(x), f64(Wg), None if b is None else f64(b), f64(W1), f64(W2))


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_step(O, w, inp, ntok):
    xs, Wg, b, W1, W2 = inp
    t0 = time.perf_counter()
    O.forward(xs[:ntok], Wg, b, W1, W2, w.k, w.cf)
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s, x, Wg, b, W1, W2):
    """The oracle as it stands, timed on the host cores on a bounded token sample."""
    import oracle as O
    inp = _oracle_inputs(w, x, Wg, b, W1, W2)
    probe = min(w.S, 256)
    c = _oracle_step(O, w, inp, probe) / probe                 # seconds per token
    ntok = int(max(64, min(w.S, budget_s / max(c, 1e-9))))
    dt = _oracle_step(O, w, inp, ntok)
    reps = 1
    # a whole workload shorter than the budget is run again until the budget is spent
    if ntok == w.S:
        more = max(0, min(19, int((budget_s - dt) / max(dt, 1e-9))))
        dt += sum(_oracle_step(O, w, inp, ntok) for _ in range(more))
        reps += more
    what = (f"first {ntok} of {w.S} tokens of the {w.name} workload (same M, H, E, k, cf; "
            f"C scaled to the sample)" if ntok < w.S else
            f"the whole {w.name} workload ({w.S} tokens), {reps} pass{'es' if reps > 1 else ''}")
    return {"value": round(reps * ntok / dt, 2), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{what}; float64 oracle forward, {dt:.1f} s; weights converted to float64 "
                      f"once, outside the timing"}


def run_reference(args, rank, world):
    w = WORKLOADS[args.workload]
    if rank != 0:
        return None
    import oracle as O
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = _oracle_inputs(w, *make_inputs(w, device=dev))
    torch.cuda.empty_cache() if dev == "cuda" else None
    probe = min(w.S, 256)
    c = _oracle_step(O, w, inp, probe) / probe
    # per-step sample sized so the whole run stays near args.ref_budget seconds
    per_step = args.ref_budget / max(1, args.steps + args.warmup)
    ntok = int(max(64, min(w.S, per_step / max(c, 1e-9))))
    for _ in range(args.warmup):
        _oracle_step(O, w, inp, ntok)
    times = [_oracle_step(O, w, inp, ntok) for _ in range(args.steps)]
    tot = sum(times)
    v = round(ntok * args.steps / tot, 2)
    return {
        "impl": "reference",
        "metric": "MoE-layer tokens/sec on 1 B200; FFN % of bf16 TC peak; dispatch/combine HBM GB/s",
        "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{w.name} (S={w.S}, M={w.M}, H={w.H}, E={w.E}, k={w.k}, cf={w.cf})",
                   "S": w.S, "M": w.M, "H": w.H, "E": w.E, "k": w.k, "capacity_factor": w.cf},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"first {ntok} of {w.S} tokens per step (same M, H, E, k, cf; "
                                   f"C scaled to the sample); float64 oracle forward"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="mid")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the CPU baseline sample")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the training-step (forward + backward) measurement")
    ap.add_argument("--eager", action="store_true",
                    help="time eager moe_forward calls instead of a CUDA-graph replay")
    args = ap.parse_args()
    if args.impl == "ours" and args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
