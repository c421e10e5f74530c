"""The allocation-free capacity entry point against the oracle and the layer's own routing (GPU).

moe_assign_slots_noalloc exists for callers that cannot call cudaMalloc, such
as a serving process whose memory pool already holds almost all of HBM, or a
runtime that routes every allocation through its own allocator.  It keeps its
scratch in a fixed device array inside the library, shared by every call.

Each case feeds it expert ids and requires, bit for bit, the slots and the
per-expert demand that the CPU oracle's capacity rule (`assign_slots`) gives
for the same ids; where the ids come from the existing entry point
(moe_route_from_logits, read back with moe_get_routing), they must also equal
that entry point's slots.  Calls run back to back, a smaller call after a
larger one, so stale scratch from an earlier call would show.  This file is
collected last; it passes alone in a fresh process as well as after the
other tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200 import _lib as L
from gshard_top_gating_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _routing_by_existing_entry(h, logits, S, E, k):
    L.moe_route_from_logits(h, S, logits)
    eidx = torch.empty(S, k, dtype=torch.int32, device="cuda")
    slot = torch.empty(S, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    L.moe_get_routing(h, eidx, None, slot, cnt)
    return eidx, slot, cnt


def _noalloc(eidx, E, k, C):
    S = eidx.shape[0]
    slot = torch.full((max(S, 1), k), -7, dtype=torch.int32, device="cuda")[:S]
    cnt = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    L.moe_assign_slots_noalloc(S, E, k, C, eidx, slot, cnt)
    torch.cuda.synchronize()
    return slot.cpu().numpy(), cnt.cpu().numpy()


def _oracle_slots(ids, E, C):
    """The oracle's rank-major capacity rule on the ids in [0, E); other ids are
    counted nowhere and get slot -1 (they are routed to no expert)."""
    ids = np.asarray(ids)
    valid = (ids >= 0) & (ids < E)
    # an invalid id is given expert E (an extra, never-reported expert), so it
    # takes no slot and no demand of a real expert
    slot, cnt = O.assign_slots(np.where(valid, ids, E), E + 1, C)
    return np.where(valid, slot, -1), cnt[:E]


def test_noalloc_slots_match_oracle_and_existing_entry_point_twice():
    E, k, cf, S_max = 24, 2, 0.8, 1500
    w = Workload("noalloc", 64, 64, 64, E, k, cf, "f32")
    _, Wg, _, W1, W2 = make_inputs(w, device="cuda")
    h = L.moe_create(S_max, 64, 64, E, k, cf, "f32", Wg, None, W1, W2)
    gen = torch.Generator(device="cuda").manual_seed(5)
    try:
        for S in (1500, 333):
            logits = torch.randn(S, E, device="cuda", generator=gen)
            logits[:, 3] += 1.5                                   # a hot expert that overflows
            eidx, slot_ref, cnt_ref = _routing_by_existing_entry(h, logits, S, E, k)
            C = L.moe_get_capacity(h, S)
            slot, cnt = _noalloc(eidx, E, k, C)
            o_slot, o_cnt = _oracle_slots(eidx.cpu().numpy(), E, C)
            assert (o_slot < 0).any() and (o_slot >= 0).any()
            assert np.array_equal(slot, o_slot) and np.array_equal(cnt, o_cnt)
            assert np.array_equal(slot, slot_ref.cpu().numpy())
            assert np.array_equal(cnt, cnt_ref.cpu().numpy())
    finally:
        L.moe_destroy(h)


def test_noalloc_top8_of_256_with_out_of_range_ids():
    E, k = 256, 8
    rng = np.random.default_rng(11)
    for S, C in ((3000, 70), (130, 3)):
        # distinct experts per token, skewed toward low ids so some overflow
        ids = np.stack([rng.choice(E, k, replace=False, p=None) for _ in range(S)]).astype(np.int32)
        ids[rng.random((S, k)) < 0.3] //= 8
        for t in range(S):                                    # keep each row's ids distinct
            seen = set()
            for r in range(k):
                while ids[t, r] in seen:
                    ids[t, r] = (ids[t, r] + 1) % E
                seen.add(int(ids[t, r]))
        bad = rng.random((S, k)) < 0.05                       # ids -1 and E are routed nowhere
        ids[bad] = np.where(rng.random(bad.sum()) < 0.5, -1, E)
        slot, cnt = _noalloc(torch.from_numpy(ids).cuda(), E, k, C)
        o_slot, o_cnt = _oracle_slots(ids, E, C)
        assert np.all(slot[bad] == -1)
        assert (o_slot >= 0).any() and ((o_slot < 0) & ~bad).any()
        assert np.array_equal(slot, o_slot) and np.array_equal(cnt, o_cnt)


def test_noalloc_empty_batch_zeroes_demand():
    cnt = torch.full((40,), 9, dtype=torch.int32, device="cuda")
    eidx = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    slot = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    L.moe_assign_slots_noalloc(0, 40, 2, 5, eidx, slot, cnt)
    torch.cuda.synchronize()
    assert torch.count_nonzero(cnt).item() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    eidx = torch.zeros(8, 2, dtype=torch.int32, device="cuda")
    out = torch.zeros(8, 2, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(256, dtype=torch.int32, device="cuda")
    with pytest.raises(L.MoeError) as ei:
        # 8 * 2^20 tokens: the local-rank table alone exceeds the 8 MiB scratch
        L.moe_assign_slots_noalloc(1 << 23, 256, 8, 10, eidx, out, cnt)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED
