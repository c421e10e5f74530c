"""Top-1 routing with the combine fused into the second expert GEMM (GPU).

On an inference handle (no moe_enable_backward) with k = 1 and bf16, the second
GEMM's epilogue stores g * row straight into the token's row of y and no combine
kernel runs.  With one choice the normalised gate is exactly 1, so y must equal,
bit for bit, the separate-combine path (a handle in training mode), and the
oracle within the bf16 tolerance; tokens whose choice was dropped get exact zeros.
The shapes take the one-CTA and CTA-pair tilings of that GEMM.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200 import _lib as L
from gshard_top_gating_b200.inputs import Workload, make_inputs
from gshard_top_gating_b200.layer import MoeLayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [
    Workload("t1_below_capacity", 3000, 256, 512, 16, 1, 1.0, "bf16"),   # below capacity
    Workload("t1_pairs", 4096, 256, 256, 8, 1, 0.5, "bf16"),             # at capacity: CTA pairs
    Workload("t1_one_cta", 1000, 192, 128, 8, 1, 1.5, "bf16", skew_bias=True),   # N = 192: one-CTA tiles
    Workload("t1_big", 20000, 1024, 1024, 64, 1, 1.0, "bf16"),
], ids=lambda w: w.name)
def test_fused_top1_equals_separate_combine(w):
    x, Wg, b, W1, W2 = make_inputs(w, device="cuda")
    inf = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    trn = MoeLayer(w.S, w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    trn.enable_backward()                                  # keeps the separate combine
    y_inf = torch.full_like(x, float("nan"))               # every row must be written
    y_trn = torch.empty_like(x)
    for _ in range(2):                                     # twice: stale tables would show
        inf(x, out=y_inf)
        trn(x, out=y_trn)
        torch.cuda.synchronize()
        assert torch.equal(y_inf, y_trn)
    assert L.moe_kernels_per_forward(inf.h, w.S) == L.moe_kernels_per_forward(trn.h, w.S) - 1
    logits = inf.logits(w.S).cpu().numpy()
    rt = O.route(logits, w.k, w.cf)
    eidx, gate, slot, cnt = (t.cpu().numpy() for t in inf.routing(w.S))
    assert np.array_equal(slot, rt.slot) and np.array_equal(eidx, rt.ids)
    assert (rt.slot < 0).any(), "the case drops some tokens"
    ref = O.outputs_for_tokens(np.arange(w.S), x.cpu(), rt.ids, rt.gates, rt.slot,
                               lambda e: (W1[e].cpu(), W2[e].cpu()))
    got = y_inf.float().cpu().numpy()
    assert np.all(got[rt.slot[:, 0] < 0] == 0.0)
    err = G.rel_err(got, ref)
    assert err <= G.TOL_Y["bf16"], err
    # the fused forward keeps no expert outputs
    with pytest.raises(L.MoeError) as ei:
        inf.expert_rows(L.MOE_BUF_Y, 0, 1)
    assert ei.value.status == L.MOE_ERR_STATE
    inf.enable_backward()
    with pytest.raises(L.MoeError) as ei:
        inf.backward(x, x)
    assert ei.value.status == L.MOE_ERR_STATE
    print(f"\n{w.name}: dropped {(rt.slot < 0).mean():.3f}, output rel err {err:.3e}")
    inf.close()
    trn.close()
