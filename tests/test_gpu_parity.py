"""CUDA path vs the oracle on small and ragged shapes, element by element (GPU).

Sizes are small enough for the full oracle but span several GEMM tiles (128
rows x 64/128/256 columns), router chunks (64 tokens) and ragged tails.
"""
import numpy as np
import pytest
import torch

from gshard_top_gating_b200.inputs import WORKLOADS, Workload, make_inputs
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def test_tiny_workload_full_oracle():
    run = G.build(WORKLOADS["tiny"])
    out, rt = G.full_check(run)
    assert rt.C == 80
    run.layer.close()


@pytest.mark.parametrize("S", [1, 2, 63, 64, 65, 129, 200, 255, 256])
def test_tiny_ragged_token_counts(S):
    run = G.build(WORKLOADS["tiny"], S=256)
    G.full_check(run, S)
    run.layer.close()


BF16_SHAPES = [
    # (S, M, H, E, k, cf) -- BN=256 / 128 / 64 paths, drops, no drops, ragged rows
    (300, 256, 512, 8, 2, 1.25),
    (300, 128, 384, 8, 2, 1.25),
    (257, 192, 320, 6, 2, 1.0),
    (500, 64, 64, 16, 2, 0.3),
    (130, 128, 256, 4, 2, 2.0),
    (400, 256, 256, 32, 4, 1.5),
    (1000, 128, 256, 64, 8, 1.25),
    (129, 128, 128, 1, 1, 1.0),       # E=1: dense FFN
    (70, 128, 256, 5, 5, 1.0),        # k = E
    (1, 128, 256, 8, 2, 1.25),
    (300, 128, 128, 200, 8, 1.25),    # router: E padded to 256, top-8
    (200, 192, 128, 100, 3, 1.0),     # router: E padded to 128
    (333, 64, 64, 33, 2, 1.0),        # router: E padded to 64
    (600, 256, 512, 4, 2, 0.5),       # experts at capacity: CTA-pair GEMMs (256-row tiles)
    (1000, 256, 256, 8, 1, 1.0),      # CTA pair, k=1, exactly at capacity
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=[str(s) for s in BF16_SHAPES])
def test_bf16_shapes_full_oracle(shape):
    S, M, H, E, k, cf = shape
    w = Workload("case", S, M, H, E, k, cf, "bf16", seed=7)
    run = G.build(w)
    G.full_check(run)
    run.layer.close()


F32_SHAPES = [(200, 64, 128, 4, 2, 1.0), (129, 128, 64, 1, 1, 1.0), (100, 64, 192, 16, 3, 0.5)]


@pytest.mark.parametrize("shape", F32_SHAPES, ids=[str(s) for s in F32_SHAPES])
def test_f32_shapes_full_oracle(shape):
    S, M, H, E, k, cf = shape
    run = G.build(Workload("case", S, M, H, E, k, cf, "f32", seed=3))
    G.full_check(run)
    run.layer.close()


def test_gate_bias_small_skewed():
    w = WORKLOADS["skewed"].with_(S=512, M=128, H=256, E=32)
    run = G.build(w)
    out, rt = G.full_check(run)
    assert (rt.slot < 0).mean() > 0.3            # hot experts overflow
    run.layer.close()


def test_all_dropped_tokens_are_zero():
    # C = 1: only the first token of each expert keeps a row
    w = Workload("drop", 256, 128, 128, 4, 2, 0.001, "bf16", seed=5)
    run = G.build(w)
    out, rt = G.full_check(run)
    assert rt.C == 1
    dropped = np.all(rt.slot < 0, axis=1)
    assert dropped.sum() > 200
    assert torch.all(out.y[torch.as_tensor(np.nonzero(dropped)[0], device="cuda")] == 0)
    run.layer.close()


def test_routing_ties_from_given_logits():
    w = Workload("ties", 300, 64, 64, 8, 2, 1.0, "f32")
    run = G.build(w)
    rng = np.random.default_rng(11)
    for E_vals in (2, 3):
        lg = rng.integers(0, E_vals, size=(300, 8)).astype(np.float32)
        lg[:5] = 0.0
        lg[5, :] = -0.0
        lg[6, ::2] = -0.0
        run.layer.route_from_logits(torch.from_numpy(lg).cuda())
        torch.cuda.synchronize()
        eidx, gate, slot, cnt = (t.cpu().numpy() for t in run.layer.routing(300))
        import oracle as O
        rt = O.route(lg, 2, 1.0)
        assert np.array_equal(eidx, rt.ids)
        assert np.array_equal(slot, rt.slot)
        assert np.array_equal(cnt, rt.cnt)
        l_aux, z = run.layer.aux_loss()
        assert abs(l_aux - rt.l_aux) <= 1e-5 * rt.l_aux
        assert abs(z - rt.z) <= 1e-5 * rt.z
    run.layer.close()


def test_empty_batch():
    from gshard_top_gating_b200 import _lib as L
    run = G.build(WORKLOADS["tiny"], S=16)
    y = torch.empty(0, 64, device="cuda")
    run.layer(run.x[:0], out=y)
    assert run.layer.aux_loss() == (0.0, 0.0)
    assert L.moe_kernels_per_forward(run.layer.h, 0) == 0
    run.layer.close()


def test_forward_is_deterministic_and_host_path_matches():
    w = Workload("det", 1000, 256, 512, 16, 2, 1.0, "bf16", seed=9)
    run = G.build(w)
    y1 = run.layer(run.x).clone()
    r1 = [t.clone() for t in run.layer.routing(1000)]
    y2 = run.layer(run.x)
    r2 = run.layer.routing(1000)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert all(torch.equal(a, b) for a, b in zip(r1, r2))
    xh = run.x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    run.layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    assert torch.equal(yh, y1.cpu())
    run.layer.close()


def test_status_errors():
    from gshard_top_gating_b200 import _lib as L
    w = WORKLOADS["tiny"]
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda", S=64)
    h = L.moe_create(64, w.M, w.H, w.E, w.k, w.cf, "f32", Wg, None, W1, W2)
    with pytest.raises(L.MoeError) as ei:
        L.moe_aux_loss(h)
    assert ei.value.status == L.MOE_ERR_STATE
    y = torch.empty_like(x)
    with pytest.raises(L.MoeError) as ei:
        L.moe_forward(h, 65, x, y)
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoeError) as ei:
        L.moe_forward(h, 4, x.data_ptr() + 4, y)
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    L.moe_forward(h, 64, x, y)
    L.moe_check(h)
    L.moe_destroy(h)


def test_bounded_wait_times_out_and_context_survives():
    from gshard_top_gating_b200 import _lib as L
    assert L.moe_selftest_wait_timeout(2000) == L.MOE_ERR_TIMEOUT
    run = G.build(Workload("after", 100, 128, 128, 4, 2, 1.0, "bf16"))
    G.full_check(run)
    run.layer.close()


def test_stage_profiling():
    from gshard_top_gating_b200 import _lib as L
    run = G.build(Workload("prof", 512, 256, 512, 8, 2, 1.0, "bf16"))
    L.moe_set_profiling(run.layer.h, True)
    run.layer(run.x)
    ms = L.moe_get_stage_times(run.layer.h)
    assert len(ms) == 6 and all(m >= 0 for m in ms)
    run.layer.close()
