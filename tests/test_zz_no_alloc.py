"""The allocation-free capacity entry point agrees with the layer's own routing (GPU).

moe_assign_slots_noalloc exists for callers that cannot call cudaMalloc, such
as a serving process whose memory pool already holds almost all of HBM, or a
runtime that routes every allocation through its own allocator.  It keeps its
scratch in a fixed device array inside the library.  This test feeds it the
expert ids that the existing entry point (moe_route_from_logits, read back with
moe_get_routing) produced, and requires the same slots and per-expert demand,
bit for bit, on two calls in a row.  The second call is smaller than the first,
so stale scratch from the first call would show.
"""
import pytest
import torch

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


def test_noalloc_slots_match_existing_entry_point_twice():
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
            slot = torch.full((S, k), -7, dtype=torch.int32, device="cuda")
            cnt = torch.full((E,), -7, dtype=torch.int32, device="cuda")
            L.moe_assign_slots_noalloc(S, E, k, C, eidx, slot, cnt)
            torch.cuda.synchronize()
            assert (slot_ref < 0).any() and (slot_ref >= 0).any()
            assert torch.equal(slot, slot_ref)
            assert torch.equal(cnt, cnt_ref)
    finally:
        L.moe_destroy(h)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    eidx = torch.zeros(8, 2, dtype=torch.int32, device="cuda")
    out = torch.zeros(8, 2, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(256, dtype=torch.int32, device="cuda")
    with pytest.raises(L.MoeError) as ei:
        # 8 * 2^20 tokens: the local-rank table alone exceeds the 8 MiB scratch
        L.moe_assign_slots_noalloc(1 << 23, 256, 8, 10, eidx, out, cnt)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED
