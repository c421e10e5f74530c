"""More CUDA-path vs oracle cases (GPU): handle reuse, host buffers, router tails.

* one handle, several forwards with different token counts (capacity, tensor
  maps and tables must follow S, nothing stale may leak between calls);
* the host-buffer forward with S < S_max;
* the tensor-core router's token tiles (64 or 128 tokens) with ragged tails,
  several K-segments (M = 576 and 1536: 9 and 24 k-blocks of 64), a gate bias
  with E padded to 256 and top-8.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200.inputs import Workload, gate_bias, make_inputs
from gshard_top_gating_b200.layer import MoeLayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def test_one_handle_many_token_counts():
    w = Workload("reuse", 1000, 256, 512, 16, 2, 0.75, "bf16", seed=21)
    run = G.build(w)
    for S in (1000, 37, 640, 1, 1000, 129):
        G.full_check(run, S)
    run.layer.close()


def test_host_buffers_smaller_batch():
    w = Workload("host", 700, 128, 256, 8, 2, 1.25, "bf16", seed=22)
    run = G.build(w)
    S = 333
    xh = run.x[:S].cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    run.layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    y_dev = run.layer(run.x[:S].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())
    G.full_check(run, S)
    run.layer.close()


ROUTER_SHAPES = [
    # (S, M, H, E, k, cf)
    (333, 256, 256, 100, 3, 1.0),     # EP = 128 -> 128-token CTAs, ragged tail of 77
    (97, 128, 128, 40, 2, 1.0),       # EP = 64  -> 64-token CTAs, ragged tail of 33
    (300, 576, 256, 24, 2, 1.25),     # 9 k-blocks: two K-segments, the last partial
    (200, 1536, 256, 8, 2, 1.25),     # 24 k-blocks: three K-segments
    (64, 256, 256, 256, 8, 1.25),     # E = 256, top-8, one CTA
    # enough tokens for 128-token CTAs with E <= 64 on 148 SMs: the 8-warp, two-per-SM
    # router; ragged last tiles whose second 64-token chunk is empty or partial
    (19001, 576, 256, 40, 2, 1.0),    # EP = 64, two K-segments, last tile 57 tokens
    (20000, 128, 128, 24, 3, 1.25),   # EP = 32, top-3, last tile 32 tokens
    (19050, 192, 128, 64, 1, 1.0),    # EP = 64, top-1, last tile 106 tokens
    (257, 128, 128, 12, 8, 1.0),      # EP = 32, top-8 of 12 (thread-per-token), one-token last tile
]


@pytest.mark.parametrize("shape", ROUTER_SHAPES, ids=[str(s) for s in ROUTER_SHAPES])
def test_router_tiles_and_segments(shape):
    S, M, H, E, k, cf = shape
    run = G.build(Workload("rt", S, M, H, E, k, cf, "bf16", seed=23))
    G.full_check(run)
    run.layer.close()


TIE_SHAPES = [
    # (S, M, H, E, k, cf)
    (300, 128, 128, 16, 4, 1.25),     # EP = 32: a thread per token, 64-token CTAs
    (19001, 128, 128, 40, 3, 1.0),    # EP = 64: 8-warp CTAs, two per SM
    (300, 128, 128, 100, 4, 1.0),     # EP = 128: a warp per token
]


@pytest.mark.parametrize("shape", TIE_SHAPES, ids=[str(s) for s in TIE_SHAPES])
def test_tensor_core_router_exact_ties(shape):
    """W_g whose odd columns repeat the even column before them: the tensor-core
    router computes both columns from the same operand values, so every token's
    logits tie in pairs, bitwise.  Top-k then has to take the lower index of a tied
    pair first; routing against the oracle on those logits stays bit-exact."""
    S, M, H, E, k, cf = shape
    w = Workload("ties_tc", S, M, H, E, k, cf, "bf16", seed=37)
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    Wg[:, 1::2] = Wg[:, 0::2]
    layer = MoeLayer(S, M, H, E, k, cf, Wg, b, W1, W2)
    run = SimpleNamespace(w=w, S=S, x=x, Wg=Wg, b=b, W1=W1, W2=W2, layer=layer)
    out = G.forward(run)
    assert np.array_equal(out.logits[:, 1::2], out.logits[:, 0::2])
    rt = G.check_routing(run, out)
    # an odd expert is chosen only after the even expert it ties with (lower index first)
    ids = out.eidx
    for r in range(k):
        e = ids[:, r]
        before = (ids[:, :r] == (e - 1)[:, None]).any(axis=1)
        assert np.all((e % 2 == 0) | before), r
    G.check_outputs(run, out, rt, np.arange(min(S, 2048)))
    layer.close()


def test_gate_bias_with_256_experts_top8():
    w = Workload("bias256", 256, 128, 128, 200, 8, 1.0, "bf16", skew_bias=True, seed=24)
    run = G.build(w)
    out, rt = G.full_check(run)
    assert (rt.slot < 0).any()                 # the bias makes low-index experts overflow
    run.layer.close()


def test_dropless_capacity_factor_keeps_everything():
    # cf = E / k gives C = S: no assignment can be dropped (the "dropless" special case)
    w = Workload("dropless", 500, 128, 256, 16, 2, 8.0, "bf16", seed=25)
    run = G.build(w)
    out, rt = G.full_check(run)
    assert rt.C == 500 and np.all(rt.slot >= 0)
    run.layer.close()


def test_host_pipeline_back_to_back_calls():
    """moe_forward_host calls issued back to back (their copies overlap the previous
    call's compute) each return exactly what a device forward of the same batch does,
    also with a device forward and different token counts in between."""
    w = Workload("pipe", 700, 128, 256, 8, 2, 1.25, "bf16", seed=26)
    run = G.build(w)
    batches = []
    for i, S in enumerate((700, 333, 700, 1, 512, 700)):
        xd = torch.roll(run.x, shifts=37 * i, dims=0)[:S].contiguous()
        batches.append((xd, xd.cpu().pin_memory(), torch.empty(S, w.M, dtype=xd.dtype).pin_memory()))
    y_mid = None
    for i, (xd, xh, yh) in enumerate(batches):
        run.layer.forward_host(xh, yh)
        if i == 2:
            y_mid = run.layer(batches[1][0])        # a device forward between host calls
    torch.cuda.synchronize()
    for xd, xh, yh in batches:
        ref = run.layer(xd)
        torch.cuda.synchronize()
        assert torch.equal(yh, ref.cpu())
    assert torch.equal(y_mid, run.layer(batches[1][0]))
    run.layer.close()


def test_cuda_graph_replay_matches_eager():
    """moe_forward captured in a CUDA graph (as the bench times it) and replayed on
    new contents of the same input buffer gives what an eager call gives."""
    w = Workload("graph", 512, 256, 512, 8, 2, 1.25, "bf16", seed=27)
    run = G.build(w)
    x = run.x.clone()
    y = torch.empty_like(x)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run.layer(x, out=y)                      # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run.layer(x, out=y)
    for shift in (0, 101, 7):
        x.copy_(torch.roll(run.x, shifts=shift, dims=0))
        graph.replay()
        torch.cuda.synchronize()
        ref = run.layer(x.clone())
        torch.cuda.synchronize()
        assert torch.equal(y, ref), shift
    del graph
    run.layer.close()
