"""Rerouting of dropped choices on the GPU against the oracle's `reroute` (GPU).

With MOE_ROUTE_REROUTE a dropped choice gets one second chance at the token's
next-ranked unchosen expert, in the capacity pass's order, into the room the pass
left.  Given the same fp32 logits the final slots, the serving experts and the
per-expert demand must equal the oracle's bit for bit; the layer output must
match the oracle's forward with the same rerouting within the usual tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200 import _lib as L
from gshard_top_gating_b200.inputs import WORKLOADS, Workload, make_inputs
from gshard_top_gating_b200.layer import MoeLayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _layer(E, k, cf, S_max, act="f32", M=64, H=64):
    w = Workload("rr", S_max, M, H, E, k, cf, act)
    _, Wg, b, W1, W2 = make_inputs(w, device="cuda", S=1)
    layer = MoeLayer(S_max, M, H, E, k, cf, Wg, b, W1, W2)
    layer.set_rerouting(True)
    return layer


def _routing(layer, S):
    eidx, gate, slot, cnt = (t.cpu().numpy() for t in layer.routing(S))
    return eidx, slot, cnt, layer.serving_experts(S).cpu().numpy()


@pytest.mark.parametrize("S,E,k,cf,skew,ties", [
    (1000, 16, 2, 1.0, 1.5, False),
    (777, 16, 2, 0.5, 0.0, True),          # tie-heavy logits
    (2000, 64, 2, 1.25, 2.0, False),
    (513, 256, 8, 0.5, 1.0, False),
    (300, 12, 8, 1.0, 1.0, False),         # k + j can exceed E: some offers have no alternative
    (129, 4, 4, 0.5, 0.5, True),           # k = E: nothing to reroute to
    (64, 40, 3, 0.3, 3.0, False),
])
def test_rerouted_slots_bit_exact_given_logits(S, E, k, cf, skew, ties):
    layer = _layer(E, k, cf, S)
    gen = torch.Generator(device="cuda").manual_seed(S + E)
    logits = torch.randn(S, E, device="cuda", generator=gen)
    if ties:
        logits = torch.round(logits * 2) / 2
    logits += skew * torch.log(1.0 / torch.arange(1, E + 1, device="cuda", dtype=torch.float32))
    layer.route_from_logits(logits.contiguous())
    eidx, slot, cnt, dest = _routing(layer, S)
    rt = O.route(logits.cpu().numpy(), k, cf, rerouting=True)
    assert np.array_equal(eidx, rt.ids)
    assert np.array_equal(cnt, rt.cnt)
    assert np.array_equal(slot, rt.slot), "final slots"
    assert np.array_equal(dest, rt.dest), "serving experts"
    print(f"\nS={S} E={E} k={k}: dropped {(rt.slot0 < 0).mean():.3f} -> {(rt.slot < 0).mean():.3f} "
          f"after rerouting")
    layer.close()


@pytest.mark.parametrize("w", [
    Workload("rr_bf16", 1500, 256, 512, 16, 2, 0.75, "bf16", skew_bias=True),
    Workload("rr_bf16_top4", 700, 128, 256, 32, 4, 0.6, "bf16", skew_bias=True),
    Workload("rr_f32", 256, 64, 256, 8, 2, 0.6, "f32", skew_bias=True),
], ids=lambda w: w.name)
def test_rerouted_forward_matches_oracle(w):
    run = G.build(w)
    run.layer.set_rerouting(True)
    out = G.forward(run)
    dest = run.layer.serving_experts(w.S).cpu().numpy()
    rt = O.route(out.logits, w.k, w.cf, rerouting=True)
    assert np.array_equal(out.eidx, rt.ids) and np.array_equal(out.slot, rt.slot)
    assert np.array_equal(dest, rt.dest) and np.array_equal(out.cnt, rt.cnt)
    assert (rt.dest != rt.ids).any(), "the case reroutes something"
    assert abs(out.l_aux - rt.l_aux) <= 1e-5 * rt.l_aux and abs(out.z - rt.z) <= 1e-5 * rt.z
    tokens = np.arange(w.S)
    ref = O.outputs_for_tokens(tokens, run.x.cpu(), rt.dest, rt.gates, rt.slot,
                               lambda e: (run.W1[e].cpu(), run.W2[e].cpu()))
    err = G.rel_err(out.y.float().cpu().numpy(), ref)
    assert err <= G.TOL_Y[w.act], err
    with_rr = L.moe_kernels_per_forward(run.layer.h, w.S)
    L.moe_set_routing_flags(run.layer.h, 0)
    assert with_rr == L.moe_kernels_per_forward(run.layer.h, w.S) + 2     # offers and their scan
    L.moe_set_routing_flags(run.layer.h, L.MOE_ROUTE_REROUTE)
    # rerouting off again: the plain layer
    run.layer.set_rerouting(False)
    out2 = G.forward(run)
    rt2 = G.check_routing(run, out2)
    assert np.array_equal(run.layer.serving_experts(w.S).cpu().numpy(), rt2.ids)
    run.layer.close()


def test_rerouted_skewed_workload_full_size():
    """The skewed workload (93% of choices dropped by the capacity pass) with rerouting:
    full routing bit-exact, outputs on 1024 sampled tokens."""
    w = WORKLOADS["skewed"]
    run = G.build(w)
    run.layer.set_rerouting(True)
    out = G.forward(run)
    dest = run.layer.serving_experts(w.S).cpu().numpy()
    rt = O.route(out.logits, w.k, w.cf, rerouting=True)
    assert np.array_equal(out.slot, rt.slot) and np.array_equal(dest, rt.dest)
    rng = np.random.default_rng(5)
    tokens = np.unique(rng.choice(w.S, 1024, replace=False))
    xs = run.x[torch.as_tensor(tokens, device="cuda")].cpu()
    ref = O.outputs_for_tokens(tokens, xs, rt.dest, rt.gates, rt.slot,
                               lambda e: (run.W1[e].cpu(), run.W2[e].cpu()))
    got = out.y[torch.as_tensor(tokens, device="cuda")].float().cpu().numpy()
    err = G.rel_err(got, ref)
    assert err <= G.TOL_Y[w.act], err
    print(f"\nskewed: kept {(rt.slot0 >= 0).mean():.4f} -> {(rt.slot >= 0).mean():.4f} of choices; "
          f"output rel err {err:.3e}")
    run.layer.close()
