"""bench.py's reference arm keeps the bench's JSON contract (CPU only).

The reference arm times the oracle on the host cores, so it runs here without a
GPU: one JSON line with the contract's keys, the oracle named as the reference.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
         "--warmup", "1", "--ref-budget", "2"],
        cwd=ROOT, capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, out
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
                "cpu_baseline"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["S"] == 256 and d["config"]["E"] == 8


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_expert_gemm_stages_take_the_slower_bound():
    """An expert GEMM is reported against the tensor peak when its flops take longer
    than its bytes at HBM bandwidth, else against HBM (few rows per active expert)."""
    b = _bench_module()
    from gshard_top_gating_b200.inputs import WORKLOADS
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    mid, skewed = WORKLOADS["mid"], WORKLOADS["skewed"]
    e = b.algorithmic(mid, 16384, 32)["ffn1"]
    assert e[0] == "gemm" and e[1] == 2.0 * 16384 * 1024 * 4096
    assert e[2] == 16384 * 1024 * 2 + 32 * 1024 * 4096 * 2 + 16384 * 4096 * 2
    bound, ach, peak, unit = b.stage_roof(e, 1e-4, pk)
    assert (bound, unit, peak) == ("tensor", "TFLOP/s", 1000.0) and abs(ach - e[1] / 1e-4 / 1e12) < 1e-9
    e = b.algorithmic(skewed, 2300, 20)["ffn1"]
    bound, ach, peak, unit = b.stage_roof(e, 1e-4, pk)
    assert (bound, unit, peak) == ("hbm", "GB/s", 5000.0) and abs(ach - e[2] / 1e-4 / 1e9) < 1e-9
    # the backward's weight gradients are written for every expert (zeros for empty ones)
    d = b.algorithmic_bwd(skewed, 2300, 20, 0, 1)["dW2"]
    assert d[2] >= skewed.E * skewed.M * skewed.H * 2
    # 5 GB in 1 ms is 5000 GB/s, the whole of this HBM peak
    assert b.stage_entry(("hbm", 5e9), 1.0, pk) == {"ms": 1.0, "GB/s": 5000.0, "frac_of_peak": 1.0,
                                                     "bound": "hbm"}


def test_reference_arm_names_the_same_workload_config():
    """Both arms print the same config dict for a workload, so the driver can pair them."""
    b = _bench_module()
    from gshard_top_gating_b200.inputs import WORKLOADS
    for name in ("tiny", "large"):
        cfg = b.workload_config(WORKLOADS[name], 1)
        assert cfg["S"] == WORKLOADS[name].S and "l2" in cfg and cfg["workload"].startswith(name)
    assert b.workload_config(WORKLOADS["large"], 1)["C"] == 2048
    assert b.workload_config(WORKLOADS["wide"], 1)["C"] == 640


def test_layer_roofline_takes_the_slower_of_tensor_and_hbm():
    """The layer's bound is max(4*A*M*H flops at the tensor peak, all stages' bytes at HBM)."""
    b = _bench_module()
    from gshard_top_gating_b200.inputs import WORKLOADS
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    w = WORKLOADS["large"]
    A = 2 * w.S
    algo = b.algorithmic(w, A, w.E)
    r = b.layer_roofline(w, A, algo, 10.0, pk)
    flops = 4.0 * A * w.M * w.H
    nbytes = sum(e[2] if e[0] == "gemm" else e[1] for e in algo.values())
    assert r["ffn_flops"] == flops and r["total_bytes"] == nbytes
    assert r["bound"] == "tensor" and abs(r["t_tensor_us"] - flops / 1e15 * 1e6) < 0.01
    assert abs(r["frac"] - flops / 1e15 / 10e-3) < 1e-4
    # few kept rows over many experts' weights: bytes dominate
    r = b.layer_roofline(WORKLOADS["skewed"], 2300, b.algorithmic(WORKLOADS["skewed"], 2300, 20), 1.0, pk)
    assert r["bound"] == "hbm" and r["t_bound_us"] == r["t_hbm_us"]
    # the capacity scan is reported as latency-bound, with no fraction of a peak
    assert b.stage_entry(b.algorithmic(w, A, w.E)["scan"], 0.05, pk)["bound"] == "latency"
