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
from gshard_top_gating_b200.ep import EPMoeLayer, ep_forward_local, ep_forward_local_peers
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
    (Workload("ep_g3_k3", 1500, 128, 256, 24, 3, 1.25, "bf16"), (500, 700, 300)),   # odd G, k = 3
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


PHASE_CASES = [
    # experts at capacity (C = 2560, n_e about 2048): both phases non-empty, CTA-pair tiles
    (Workload("ep2_sat", 8192, 256, 512, 8, 2, 1.25, "bf16"), (3000, 1000, 2500, 1692)),
    (Workload("ep2_sat_full", 4096, 256, 256, 8, 2, 1.0, "bf16"), (2048, 2048)),
    # below capacity, one-CTA tiles; some experts above 256 rows, some below
    (Workload("ep2_skewed", 4096, 128, 256, 16, 2, 2.0, "bf16", skew_bias=True), (1000, 1100, 996, 1000)),
    # n_e about 128: every row in phase 1, phase 0 empty
    (Workload("ep2_top8", 1024, 128, 256, 64, 8, 1.25, "bf16"), (128,) * 8),
    # odd G, k = 3, some experts past the split
    (Workload("ep2_g3_k3", 6000, 128, 256, 12, 3, 1.0, "bf16"), (2500, 1000, 2500)),
]


@pytest.mark.parametrize("w,shards", PHASE_CASES, ids=[c[0].name for c in PHASE_CASES])
def test_ep_two_phases_equal_one_phase_bit_for_bit(w, shards):
    """Exchanges in two phases (split by expert slot, so that they can overlap the
    expert GEMMs) give the one-phase forward's routing, outputs and losses exactly."""
    G = len(shards)
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    El = w.E // G
    cuts = np.cumsum((0,) + shards)
    xs = [x[cuts[g]:cuts[g + 1]].contiguous() for g in range(G)]
    Ws = [(W1[g * El:(g + 1) * El].contiguous(), W2[g * El:(g + 1) * El].contiguous()) for g in range(G)]
    res = {}
    for phases in (1, 2):
        layers = [EPMoeLayer(G, g, max(shards[g], 1), w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, *Ws[g],
                             phases=phases) for g in range(G)]
        ys = ep_forward_local(layers, xs)
        torch.cuda.synchronize()
        parts = [layer.routing() for layer in layers]
        res[phases] = (torch.cat(ys), torch.cat([p[0] for p in parts]), torch.cat([p[2] for p in parts]),
                       [layer.aux_loss() for layer in layers], [layer.send_rows for layer in layers])
        for layer in layers:
            layer.close()
    y1, e1, s1, a1, _ = res[1]
    y2, e2, s2, a2, send2 = res[2]
    assert torch.equal(e1, e2) and torch.equal(s1, s2)
    assert torch.equal(y1, y2)
    assert a1 == a2
    moved0 = sum(int(s[0].sum()) for s in send2)
    moved1 = sum(int(s[1].sum()) for s in send2)
    print(f"\n{w.name}: rows in phase 0 / 1: {moved0} / {moved1}")
    if w.name.startswith("ep2_sat"):
        assert moved0 > 0 and moved1 > 0


@pytest.mark.parametrize("w,shards", CASES, ids=[c[0].name for c in CASES])
def test_ep_over_peer_memory_equals_the_all_to_all(w, shards):
    """The pack storing rows straight into the owners' receive buffers and the combine
    reading them there (one device standing in for peer memory) give the all-to-all
    forward's routing, outputs and losses bit for bit."""
    G = len(shards)
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    El = w.E // G
    cuts = np.cumsum((0,) + shards)
    xs = [x[cuts[g]:cuts[g + 1]].contiguous() for g in range(G)]
    Ws = [(W1[g * El:(g + 1) * El].contiguous(), W2[g * El:(g + 1) * El].contiguous()) for g in range(G)]
    res = []
    for fwd in (ep_forward_local, ep_forward_local_peers):
        layers = [EPMoeLayer(G, g, max(shards[g], 1), w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, *Ws[g])
                  for g in range(G)]
        for _ in range(2):                     # twice: the second forward reuses every buffer
            ys = fwd(layers, xs)
        torch.cuda.synchronize()
        parts = [layer.routing() for layer in layers]
        res.append((torch.cat(ys), torch.cat([p[0] for p in parts]), torch.cat([p[2] for p in parts]),
                    [layer.aux_loss() for layer in layers]))
        for layer in layers:
            layer.close()
    (y1, e1, s1, a1), (y2, e2, s2, a2) = res
    assert torch.equal(e1, e2) and torch.equal(s1, s2)
    assert torch.equal(y1, y2)
    assert a1 == a2


def test_ep_peer_memory_arguments():
    from gshard_top_gating_b200 import _lib as L
    w = Workload("ep_peer_args", 256, 64, 64, 8, 2, 1.0, "bf16")
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    layer = EPMoeLayer(2, 0, 128, 256, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1[:4].contiguous(), W2[:4].contiguous())
    st = layer.route(x[:128].contiguous()).cpu().numpy()
    stats = np.stack([st, st])
    with pytest.raises(L.MoeError) as ei:      # no peers set
        layer.dispatch_to_peers(stats, x[:128].contiguous())
    assert ei.value.status == L.MOE_ERR_STATE
    other = torch.empty_like(layer.recvbuf)
    with pytest.raises(L.MoeError) as ei:      # a null or misaligned buffer
        layer.set_peers([layer.recvbuf.data_ptr(), 0])
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoeError) as ei:
        layer.set_peers([layer.recvbuf.data_ptr(), other.data_ptr() + 2])
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    layer.set_peers([layer.recvbuf.data_ptr(), other.data_ptr()])
    with pytest.raises(L.MoeError) as ei:      # nothing planned yet
        layer.combine_from_peers()
    assert ei.value.status == L.MOE_ERR_STATE
    layer.dispatch_to_peers(stats, x[:128].contiguous())
    layer.experts()
    with pytest.raises(L.MoeError) as ei:      # the rows went to the peers' buffers
        layer.combine()
    assert ei.value.status == L.MOE_ERR_STATE
    layer.combine_from_peers()
    layer.dispatch(stats, x[:128].contiguous())
    with pytest.raises(L.MoeError) as ei:      # and now to the send buffer
        layer.combine_from_peers()
    assert ei.value.status == L.MOE_ERR_STATE
    L.moe_ep_set_phases(layer.h, 2)            # peers take one phase
    layer.route(x[:128].contiguous())
    with pytest.raises(L.MoeError) as ei:
        layer.dispatch_to_peers(stats, x[:128].contiguous())
    assert ei.value.status == L.MOE_ERR_STATE
    torch.cuda.synchronize()
    layer.close()


def test_ep_large_workload_over_eight_ranks_bit_exact():
    """The large workload (65536 tokens, 64 experts at capacity) split over 8 emulated
    ranks, in all three forms (all-to-all with one and two phases, peer memory), gives
    the one-device layer's output bit for bit."""
    from gshard_top_gating_b200.inputs import WORKLOADS
    w = WORKLOADS["large"]
    G = 8
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    one = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    y1 = one(x)
    torch.cuda.synchronize()
    one.close()
    El, Sg = w.E // G, w.S // G
    xs = [x[g * Sg:(g + 1) * Sg].contiguous() for g in range(G)]
    for phases, fwd in ((1, ep_forward_local), (2, ep_forward_local), (1, ep_forward_local_peers)):
        layers = [EPMoeLayer(G, g, Sg, w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b,
                             W1[g * El:(g + 1) * El].contiguous(), W2[g * El:(g + 1) * El].contiguous(),
                             phases=phases) for g in range(G)]
        ys = fwd(layers, xs)
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(ys), y1), (phases, fwd.__name__)
        for layer in layers:
            layer.close()
        del layers, ys
        torch.cuda.empty_cache()


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


def test_ep_phase_arguments():
    from gshard_top_gating_b200 import _lib as L
    w = Workload("ep_args", 256, 64, 64, 8, 2, 1.0, "f32")
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    layer = EPMoeLayer(2, 0, 128, 256, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1[:4].contiguous(), W2[:4].contiguous())
    with pytest.raises(L.MoeError) as ei:      # the FFMA GEMMs take no row base: one phase only
        L.moe_ep_set_phases(layer.h, 2)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED
    for bad in (0, 3):
        with pytest.raises(L.MoeError) as ei:
            L.moe_ep_set_phases(layer.h, bad)
        assert ei.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoeError) as ei:      # no plan yet
        layer.experts_phase(0)
    assert ei.value.status == L.MOE_ERR_STATE
    st = layer.route(x[:128].contiguous()).cpu().numpy()
    layer.dispatch(np.stack([st, st]), x[:128].contiguous())
    with pytest.raises(L.MoeError) as ei:      # phase out of range
        layer.experts_phase(1)
    assert ei.value.status == L.MOE_ERR_INVALID_ARG
    layer.close()


def test_ep_forward_dist_one_rank_nccl():
    """The torch.distributed driver (all-gather of stats, two all_to_all_single) in a
    one-rank NCCL group equals the one-device layer; no rank waits on another."""
    import os
    import socket
    import torch.distributed as dist
    from datetime import timedelta
    from gshard_top_gating_b200.ep import ep_forward_dist
    w = Workload("ep_dist1", 4096, 256, 256, 8, 2, 1.0, "bf16")      # n_e about 1024: both phases used
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        one = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
        y1 = one(x)
        lb, zb = one.aux_loss()
        for phases in (1, 2):                  # two phases: asynchronous exchanges per phase
            layer = EPMoeLayer(1, 0, w.S, w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2, phases=phases)
            y = ep_forward_dist(layer, x)
            torch.cuda.synchronize()
            assert torch.equal(y, y1), phases
            la, za = layer.aux_loss()
            assert abs(la - lb) <= 1e-5 * lb and abs(za - zb) <= 1e-5 * zb
            layer.close()
        # over peer memory: one rank's own receive buffer is its only peer
        from gshard_top_gating_b200.ep import ep_forward_dist_peers
        layer = EPMoeLayer(1, 0, w.S, w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
        layer.set_peers([layer.recvbuf.data_ptr()])
        y = ep_forward_dist_peers(layer, x)
        torch.cuda.synchronize()
        assert torch.equal(y, y1)
        layer.close()
        one.close()
    finally:
        dist.destroy_process_group()
