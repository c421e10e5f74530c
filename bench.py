"""Benchmark of the GShard MoE layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload large]

A step is one whole layer forward (router, capacity scan, dispatch, two grouped
expert GEMMs, combine, losses) over one batch of synthetic tokens already
resident in HBM.  The headline workload is the largest single-GPU
configuration, "large" (S=65536 tokens, M=2048, H=8192, E=64, top-2, capacity
factor 1.0, bf16).  Workloads whose token batch fits in L2 get a 256 MB write (an
L2 flush) before every timed step; those whose inputs are larger than L2 (large
and wide: x of 268 and 235 MB, expert weights of GBs) are timed without one, and
`config.l2` says which.  Each step is timed with CUDA events on the launching
stream; the sum over the K steps is the timed region.  The other four workloads are timed the same way
in the same run and reported under "per_workload" (--workload-only skips them).

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
L2_BYTES = 126 * 1024 * 1024          # B200 L2 cache


def inputs_exceed_l2(w) -> bool:
    """The token batch alone is larger than L2 (and the expert weights far larger), so no
    step can find the previous step's inputs in L2: such workloads are timed without a
    flush; the others get a 256 MB write before every timed step."""
    s = 2 if w.act == "bf16" else 4
    return w.S * w.M * s > L2_BYTES and w.E * w.M * w.H * s * 2 > L2_BYTES
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
    with a kept row): ("hbm", bytes), ("latency", bytes) for a stage whose bytes are
    too few to be bound by HBM, or ("gemm", flops, bytes) for an expert GEMM, whose
    bytes are its operands read once (the active experts' weights) and its result
    written once."""
    s = 2 if w.act == "bf16" else 4
    S, M, H, E, k = w.S, w.M, w.H, w.E, w.k
    wts = n_active * M * H * s
    nchunk = (S + 63) // 64
    return {
        "router": ("hbm", S * M * s + 4 * M * E + S * E * 4 + S * k * 12),
        # chunk histograms read, their prefix offsets written, loss partials read
        "scan": ("latency", 2 * k * nchunk * E * 4 + nchunk * (E + 1) * 4),
        "dispatch": ("hbm", (S + A) * M * s),
        "ffn1": ("gemm", 2.0 * A * M * H, A * M * s + wts + A * H * s),
        "ffn2": ("gemm", 2.0 * A * M * H, A * H * s + wts + A * M * s),
        "combine": ("hbm", (A + S) * M * s + S * k * 12),
    }


def layer_roofline(w, A, algo, ms_per_step, pk):
    """The layer's bound: its expert-FFN flops (4*A*M*H) at the bf16 tensor peak or
    the total algorithmic bytes of all its stages at the HBM peak, whichever takes
    longer; frac = that time over the measured step."""
    flops = 4.0 * A * w.M * w.H
    nbytes = sum(e[2] if e[0] == "gemm" else e[1] for e in algo.values())
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    t = max(t_tc, t_hbm)
    out = {"bound": "tensor" if t_tc >= t_hbm else "hbm", "ffn_flops": flops, "total_bytes": nbytes,
           "t_tensor_us": round(t_tc * 1e6, 2), "t_hbm_us": round(t_hbm * 1e6, 2),
           "t_bound_us": round(t * 1e6, 2), "ms_per_step": round(ms_per_step, 5),
           "frac": round(t / (ms_per_step / 1e3), 4),
           "peaks": "bf16 burst and HBM copy"}
    if pk.get("bf16_tflops_sustained"):
        t_s = max(flops / (pk["bf16_tflops_sustained"] * 1e12), t_hbm)
        out["frac_of_sustained"] = round(t_s / (ms_per_step / 1e3), 4)
    return out


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
    rows per expert streams weights faster than it can use the tensor cores).  A
    latency-bound stage reports its bytes per second with no peak."""
    if entry[0] == "latency":
        return "latency", entry[1] / seconds / 1e9, None, "GB/s"
    if entry[0] == "gemm":
        flops, nbytes = entry[1], entry[2]
        if flops / (pk["bf16_tflops"] * 1e12) >= nbytes / (pk["hbm_gbs"] * 1e9):
            return "tensor", flops / seconds / 1e12, pk["bf16_tflops"], "TFLOP/s"
        return "hbm", nbytes / seconds / 1e9, pk["hbm_gbs"], "GB/s"
    return "hbm", entry[1] / seconds / 1e9, pk["hbm_gbs"], "GB/s"


def stage_entry(entry, ms, pk):
    b_, ach, peak, unit = stage_roof(entry, ms / 1e3, pk)
    return {"ms": round(ms, 4), unit: round(ach, 1),
            "frac_of_peak": round(ach / peak, 4) if peak else None, "bound": b_}


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


def measure_backward(args, w, weights, x, y, flush, stream, pk, pk_kind, A, n_e):
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
    if inputs_exceed_l2(w):
        flush = None
    n = max(3, min(args.steps, 50))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    for i in range(n):
        if flush is not None:
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
        if flush is not None:
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
    timed = {k_: t for k_, t in stage_ms.items() if algo[k_][0] != "latency"}
    dom = max(timed, key=lambda k_: timed[k_])
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
                     "peak_source": f"{pk_kind}, burst" if b_ == "tensor" else pk_kind,
                     "frac_of_sustained": (round(ach / pk["bf16_tflops_sustained"], 4)
                                           if b_ == "tensor" and pk.get("bf16_tflops_sustained") else None)},
        "stages": stages,
        "gpu_launches": launches,
    }


def workload_config(w, world):
    """The workload as both arms name it (same keys and values on the reference arm)."""
    return {"workload": f"{w.name} (S={w.S}, M={w.M}, H={w.H}, E={w.E}, k={w.k}, cf={w.cf})",
            "S": w.S, "M": w.M, "H": w.H, "E": w.E, "k": w.k, "capacity_factor": w.cf,
            "C": math.ceil(w.cf * w.k * w.S / w.E),
            "l2": (f"inputs larger than L2 (x {w.S * w.M * (2 if w.act == 'bf16' else 4) / 2**20:.0f} MiB, "
                   f"expert weights {w.E * w.M * w.H * (2 if w.act == 'bf16' else 4) * 2 / 2**30:.1f} GiB, "
                   f"L2 126 MiB): no flush" if inputs_exceed_l2(w)
                   else "flushed before every timed step (256 MB write)"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def capture_step(layer, x, y, dev, eager):
    """A CUDA graph of one moe_forward (its six kernels and their programmatic
    dependencies), or None to time eager calls; with the launch note."""
    if eager:
        return None, "eager moe_forward"
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
        return graph, "CUDA graph of moe_forward"
    except Exception as exc:            # capture unsupported: time eager calls instead
        torch.cuda.synchronize()
        return None, f"eager moe_forward (graph capture failed: {type(exc).__name__})"


def time_steps(step, flush, stream, steps, world):
    """K steps (L2 flushed before each when `flush` is a buffer), device time per step;
    (total ms over ranks, t0, t1)."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.monotonic()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.monotonic()
    barrier(world)
    total = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)), world)
    return total, t0, t1


def stage_times(layer, x, y, flush, steps):
    """Per-stage device times: events the library records on the stream between its kernels."""
    from gshard_top_gating_b200 import _lib as L
    L.moe_set_profiling(layer.h, True)
    per = [[] for _ in STAGES]
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        layer(x, out=y)
        for j, t in enumerate(L.moe_get_stage_times(layer.h)):
            per[j].append(t)
    L.moe_set_profiling(layer.h, False)
    return {n: statistics.mean(v) for n, v in zip(STAGES, per)}


def measure_workload(args, w, dev, world, flush, pk, pk_kind, headline):
    """Time one workload's layer forward.  The headline workload also gets the clock
    record, the end-to-end host-buffer number, the training step and the CPU baseline."""
    from gshard_top_gating_b200 import _lib as L
    from gshard_top_gating_b200.layer import MoeLayer
    x, Wg, b, W1, W2 = make_inputs(w, device=dev)
    layer = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    if inputs_exceed_l2(w):
        flush = None
    for _ in range(args.warmup):
        layer(x, out=y)
    torch.cuda.synchronize()
    _, _, slot, cnt = layer.routing(w.S)
    C = layer.capacity(w.S)
    n_e = torch.clamp(cnt.long(), max=C)
    A = int(n_e.sum().item())
    n_active = int((n_e > 0).sum().item())
    graph, launch_note = capture_step(layer, x, y, dev, args.eager)

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer(x, out=y)

    for _ in range(2):
        step()
    torch.cuda.synchronize()

    clk = ClockSampler(dev.index or 0).__enter__() if headline else None
    total_ms, t_begin, t_end = time_steps(step, flush, stream, args.steps, world)
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.S, args.steps, total_ms, world)
    stage_ms = stage_times(layer, x, y, flush, args.steps)

    algo = algorithmic(w, A, n_active)
    stages = {n: stage_entry(algo[n], stage_ms[n], pk) for n in STAGES if stage_ms[n] > 0}
    if w.act == "bf16":
        # the dominant stage among those with a roofline (a latency-bound stage has none)
        timed = {n: t for n, t in stage_ms.items() if algo[n][0] != "latency"}
        dom = max(timed, key=lambda n: timed[n])
        bound, achieved, peak, unit = stage_roof(algo[dom], stage_ms[dom] / 1e3, pk)
        roof = {"bound": bound, "kernel": dom, "achieved": round(achieved, 2), "peak": peak,
                "unit": unit, "frac": round(achieved / peak, 4), "traffic": ncu_traffic(dom, w.name),
                "peak_source": f"{pk_kind}, burst" if bound == "tensor" else pk_kind,
                "frac_of_sustained": (round(achieved / pk["bf16_tflops_sustained"], 4)
                                      if bound == "tensor" and pk.get("bf16_tflops_sustained") else None),
                "layer": layer_roofline(w, A, algo, ms_per_step, pk)}
    else:
        roof = {"bound": "latency", "note": "fp32 activations on FFMA kernels: a parity "
                "configuration, bound by launch latency, with no roofline target"}
    out = {"value": round(value, 1), "unit": "tokens/s", "ms_per_step": round(ms_per_step, 5),
           "dtype": w.act, "config": workload_config(w, world),
           "run": {"kept_assignments": A, "active_experts": n_active, "launch": launch_note},
           "roofline": roof, "stages": stages,
           "gpu_launches": args.steps * L.moe_kernels_per_forward(layer.h, w.S)}
    if not headline:
        layer.close()
        return out

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
    del xh, yh

    # clocks: the timed region itself when it held enough samples, else a soak of
    # the same forward right after it (the timed region was too short to sample)
    if clk.count(t_begin, t_end) >= 3:
        clocks = clk.summary(t_begin, t_end, "timed region")
    else:
        s0 = time.monotonic()
        while time.monotonic() - s0 < 1.5:
            for _ in range(5):
                if flush is not None:
                    flush.zero_()
                step()
            torch.cuda.synchronize()
        clocks = clk.summary(s0, time.monotonic(),
                             "1.5 s soak of the same step right after the timed region")
    clk.__exit__()
    del graph

    out["e2e"] = {"value": round(job_throughput(w.S, args.steps, e2e_ms, world), 1), "unit": "tokens/s",
                  "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                  "ms_per_step": round(e2e_ms / args.steps, 4), "copies_alone": copies}
    out["clocks"] = clocks
    out["train_step"] = (None if args.no_backward
                         else measure_backward(args, w, (Wg, b, W1, W2), x, y, flush, stream, pk, pk_kind, A, n_e))
    layer.close()
    out["_inputs"] = (x, Wg, b, W1, W2)
    return out


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MB > L2
    pk, pk_kind = peaks()
    w = WORKLOADS[args.workload]
    head = measure_workload(args, w, dev, world, flush, pk, pk_kind, headline=True)
    x, Wg, b, W1, W2 = head.pop("_inputs")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_budget, x, Wg, b, W1, W2)
    del x, Wg, b, W1, W2
    torch.cuda.empty_cache()

    per = {}
    if not args.workload_only:
        for name, wl in WORKLOADS.items():
            if name == w.name:
                continue
            per[name] = measure_workload(args, wl, dev, world, flush, pk, pk_kind, headline=False)
            torch.cuda.empty_cache()

    line = {
        "metric": "MoE-layer tokens/sec on 1 B200; FFN % of bf16 TC peak; dispatch/combine HBM GB/s",
        "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.act, "data": "synthetic",
        "config": head["config"], "run": head["run"],
        "roofline": head["roofline"], "stages": head["stages"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        "cpu_baseline": cpu, "train_step": head["train_step"],
        "per_workload": per,
    }
    return line


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """The oracle's forward over the first ntok tokens of a workload, as a batch of
    their own (C scaled to the sample): gate logits, routing, and every sampled
    token's output through its kept experts (`outputs_for_tokens`).

    The expert weights are handed to the oracle one expert at a time in float64;
    fetching and converting them is timed apart and left out of the oracle's time.
    """

    def __init__(self, w, x, Wg, b, W1, W2):
        import numpy as np
        f64 = lambda t: None if t is None else t.detach().to("cpu", torch.float64).numpy()
        self.w = w
        self.x = x
        self.Wg, self.b = f64(Wg), f64(b)
        self.W1, self.W2 = W1, W2
        self.np = np

    def run(self, ntok):
        import oracle as O
        w = self.w
        fetch = [0.0]

        def expert_weights(e):
            t0 = time.perf_counter()
            pair = (self.W1[e].to(torch.float64).cpu().numpy(), self.W2[e].to(torch.float64).cpu().numpy())
            fetch[0] += time.perf_counter() - t0
            return pair

        t0 = time.perf_counter()
        xs = self.x[:ntok].to(torch.float64).cpu().numpy()
        fetch[0] += time.perf_counter() - t0
        t0 = time.perf_counter()
        logits = O.gate_logits(xs, self.Wg, self.b)
        rt = O.route(logits, w.k, w.cf)
        O.outputs_for_tokens(self.np.arange(ntok), xs, rt.ids, rt.gates, rt.slot, expert_weights)
        return time.perf_counter() - t0 - fetch[0]


def _sized_runs(sample, budget_s, S, probe=64, max_passes=20):
    """Oracle passes on a token sample sized to about budget_s seconds of oracle time:
    a probe pass sizes the sample; a whole workload shorter than the budget is run
    again (at most max_passes).  Returns (tokens per pass, passes, seconds)."""
    probe = min(S, probe)
    c = sample.run(probe) / probe
    ntok = int(max(probe, min(S, budget_s / max(c, 1e-9))))
    dt = sample.run(ntok)
    if dt < 0.5 * budget_s and ntok < S:        # the probe's fixed costs overstated a token's cost
        ntok = int(min(S, ntok * budget_s / max(dt, 1e-9)))
        dt = sample.run(ntok)
    reps = 1
    if ntok == S:
        more = max(0, min(max_passes - 1, int((budget_s - dt) / max(dt, 1e-9))))
        dt += sum(sample.run(ntok) for _ in range(more))
        reps += more
    return ntok, reps, dt


def cpu_baseline(w, budget_s, x, Wg, b, W1, W2):
    """The oracle as it stands, timed on the host cores on a bounded token sample: with
    every BLAS thread, and with one thread."""
    sample = OracleSample(w, x, Wg, b, W1, W2)

    def describe(ntok, reps, dt):
        what = (f"first {ntok} of {w.S} tokens of the {w.name} workload as their own batch "
                f"(same M, H, E, k, cf; C scaled to the sample)" if ntok < w.S else
                f"the whole {w.name} workload ({w.S} tokens), {reps} pass{'es' if reps > 1 else ''}")
        return (f"{what}; float64 oracle forward (gate logits, routing, outputs of every sampled "
                f"token), {dt:.1f} s of oracle time; each expert's weights fetched and converted "
                f"to float64 outside that time")

    ntok, reps, dt = _sized_runs(sample, budget_s, w.S)
    out = {"value": round(reps * ntok / dt, 2), "unit": "tokens/s", "cores": _blas_threads(),
           "kind": "oracle", "sample": describe(ntok, reps, dt)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, r1, d1 = _sized_runs(sample, budget_s / 2, w.S, probe=16, max_passes=5)
        out["single_thread"] = {"value": round(r1 * n1 / d1, 2), "unit": "tokens/s", "cores": 1,
                                "sample": describe(n1, r1, d1)}
    except ImportError:
        out["single_thread"] = None
    return out


def run_reference(args, rank, world):
    w = WORKLOADS[args.workload]
    if rank != 0:
        return None
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    sample = OracleSample(w, *make_inputs(w, device=dev))
    probe = min(w.S, 64)
    c = sample.run(probe) / probe
    # per-step sample sized so the whole run stays near args.ref_budget seconds
    per_step = args.ref_budget / max(1, args.steps + args.warmup)
    ntok = int(max(min(w.S, 16), min(w.S, per_step / max(c, 1e-9))))
    for _ in range(args.warmup):
        sample.run(ntok)
    times = [sample.run(ntok) for _ in range(args.steps)]
    tot = sum(times)
    v = round(ntok * args.steps / tot, 2)
    return {
        "impl": "reference",
        "metric": "MoE-layer tokens/sec on 1 B200; FFN % of bf16 TC peak; dispatch/combine HBM GB/s",
        "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"first {ntok} of {w.S} tokens per step as their own batch "
                                   f"(same M, H, E, k, cf; C scaled to the sample); float64 oracle "
                                   f"forward; each expert's weights fetched and converted to "
                                   f"float64 outside the timed oracle work"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="large",
                    help="the headline workload (default: large, the largest single-GPU one)")
    ap.add_argument("--workload-only", action="store_true",
                    help="time the headline workload alone (no per_workload lines)")
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
