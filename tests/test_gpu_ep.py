"""Expert-parallel forward, G ranks emulated on one GPU (GPU).

Each rank is its own library handle with its block of tokens and its E/G experts;
the exchanges between them are one device copy per (source, destination) block
(`ep_forward_local`), the bytes an all-to-all would move.  No kernel of one rank
waits on another's.  The concatenated result must be the one-device layer's on
the whole batch:
  - routing (expert ids, global slots, drops) bit-exact against the oracle routing
    the GPU's own fp32 logits, and equal to the single-GPU handle's;
  - outputs within the layer's tolerance of the oracle, on every token;
  - l_aux and z within 1e-5 of the oracle on the same logits.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200.ep import EPMoeLayer, ep_forward_local
from gshard_top_gating_b200.inputs import Workload, make_inputs
from gshard_top_gating_b200.layer import MoeLayer
from tests import gpu_helpers as Gh

pytestmark = pytest.mark.gpu

CASES = [
    # workload, shards (tokens per rank)
    (Workload("ep_bf16", 2048, 256, 512, 16, 2, 1.0, "bf16"), (1024, 1024)),
    (Workload("ep_bf16_g4", 2048, 256, 512, 16, 2, 1.0, "bf16"), (512, 700, 300, 536)),
    (Workload("ep_top8", 1024, 128, 256, 64, 8, 1.25, "bf16"), (128,) * 8),
    (Workload("ep_skewed", 1536, 128, 256, 32, 2, 1.25, "bf16", skew_bias=True), (400, 0, 600, 536)),
    (Workload("ep_sat", 4096, 256, 256, 8, 2, 1.0, "bf16"), (2048, 2048)),      # experts at capacity
    (Workload("ep_f32", 256, 64, 256, 8, 2, 1.25, "f32"), (100, 156)),
]


@pytest.mark.parametrize("w,shards", CASES, ids=[c[0].name for c in CASES])
def test_ep_emulated_ranks_equal_one_device(w, shards):
    G = len(shards)
    assert sum(shards) == w.S and w.E % G == 0
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    El = w.E // G
    cuts = np.cumsum((0,) + shards)
    layers = [EPMoeLayer(G, g, max(shards[g], 1), w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b,
                         W1[g * El:(g + 1) * El].contiguous(), W2[g * El:(g + 1) * El].contiguous())
              for g in range(G)]
    xs = [x[cuts[g]:cuts[g + 1]].contiguous() for g in range(G)]
    for rep in range(2):                       # twice: the second forward reuses every buffer
        ys = ep_forward_local(layers, xs)
        torch.cuda.synchronize()
        y = torch.cat(ys).float().cpu().numpy()
        parts = [layer.routing() for layer in layers]
        eidx = torch.cat([p[0] for p in parts]).cpu().numpy()
        gate = torch.cat([p[1] for p in parts]).cpu().numpy()
        slot = torch.cat([p[2] for p in parts]).cpu().numpy()
        logits = torch.cat([p[4] for p in parts]).cpu().numpy()
        rt = O.route(logits, w.k, w.cf)
        assert np.array_equal(eidx, rt.ids), "expert ids"
        assert np.array_equal(slot, rt.slot), "global slots / drops"
        assert np.all(np.abs(gate - rt.gates) <= 2e-6 * np.abs(rt.gates) + 1e-9)
        ref = O.outputs_for_tokens(np.arange(w.S), x.cpu(), rt.ids, rt.gates, rt.slot,
                                   lambda e: (W1[e].cpu(), W2[e].cpu()))
        err = Gh.rel_err(y, ref)
        assert err <= Gh.TOL_Y[w.act], err
        assert np.all(y[np.all(rt.slot < 0, axis=1)] == 0.0)
        for layer in layers:
            l_aux, z = layer.aux_loss()
            assert abs(l_aux - rt.l_aux) <= 1e-5 * rt.l_aux and abs(z - rt.z) <= 1e-5 * rt.z
    # the single-GPU layer on the concatenated batch: same logits, routing and outputs
    one = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y1 = one(x)
    e1, g1, s1, _ = (t.cpu().numpy() for t in one.routing(w.S))
    l1 = one.logits(w.S).cpu().numpy()
    torch.cuda.synchronize()
    assert Gh.rel_err(logits, l1) <= 1e-6
    same = bool(np.array_equal(l1, logits))
    if same:                                   # identical logits route identically
        assert np.array_equal(e1, eidx) and np.array_equal(s1, slot)
    d = float(np.abs(y1.float().cpu().numpy() - y).max())
    print(f"\n{w.name} G={G}: output rel err {err:.3e}, dropped {(slot < 0).mean():.3f}, "
          f"logits bitwise equal to one device: {same}, max |EP - one device| {d:.3e}")
    assert Gh.rel_err(y, y1.float().cpu().numpy()) <= Gh.TOL_Y[w.act]
    one.close()
    for layer in layers:
        layer.close()


def test_ep_rejects_a_plan_from_inconsistent_stats():
    w = Workload("ep_bad", 256, 64, 64, 8, 2, 1.0, "bf16")
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    layer = EPMoeLayer(2, 0, 128, 256, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1[:4].contiguous(), W2[:4].contiguous())
    st = layer.route(x[:128].contiguous()).cpu().numpy()
    from gshard_top_gating_b200 import _lib as L
    with pytest.raises(L.MoeError) as ei:      # rank 0's own token count must match its route
        bad = np.stack([st, st]); bad[0, -1] = 127
        layer.dispatch(bad, x[:128].contiguous())
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoeError):            # counts that are not integers
        bad = np.stack([st, st]); bad[1, 0] += 0.5
        layer.dispatch(bad, x[:128].contiguous())
    layer.close()


def test_ep_forward_dist_one_rank_nccl():
    """The torch.distributed driver (all-gather of stats, two all_to_all_single) in a
    one-rank NCCL group equals the one-device layer; no rank waits on another."""
    import os
    import socket
    import torch.distributed as dist
    from datetime import timedelta
    from gshard_top_gating_b200.ep import ep_forward_dist
    w = Workload("ep_dist1", 1024, 256, 256, 16, 2, 1.0, "bf16")
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        layer = EPMoeLayer(1, 0, w.S, w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
        y = ep_forward_dist(layer, x)
        one = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
        y1 = one(x)
        torch.cuda.synchronize()
        assert torch.equal(y, y1)
        la, za = layer.aux_loss()
        lb, zb = one.aux_loss()
        assert abs(la - lb) <= 1e-5 * lb and abs(za - zb) <= 1e-5 * zb
        one.close()
        layer.close()
    finally:
        dist.destroy_process_group()
