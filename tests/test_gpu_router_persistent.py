"""The persistent tensor-core router (E <= 64 and at least four 64-token chunks per SM) (GPU).

Each SM's CTA owns a contiguous range of chunks and walks it in 128-token tiles,
the last possibly a single chunk; routing of one tile overlaps the next tiles'
loads and MMAs.  Token counts here give ranges of odd and even chunk counts, a
partial last chunk, one to four K-segments of 512, and E = 32, 40 and 64: the
routing must be bit-exact against the oracle on the GPU's logits, the logits
within 1e-5 of the oracle's float64 product, the losses within 1e-5.
"""
import numpy as np
import pytest
import torch

from gshard_top_gating_b200.inputs import Workload
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [
    Workload("p_e64", 40000, 256, 64, 64, 2, 1.0, "bf16"),
    Workload("p_e32_top8_bias", 38401, 128, 64, 32, 8, 1.25, "bf16", skew_bias=True),
    Workload("p_e40_k3_4seg", 50003, 2048, 64, 40, 3, 1.0, "bf16"),
    Workload("p_e64_top1", 65536, 1024, 64, 64, 1, 1.5, "bf16"),
    Workload("p_e64_1seg_tail", 47999, 512, 128, 64, 2, 0.75, "bf16", skew_bias=True),
], ids=lambda w: w.name)
def test_persistent_router_parity(w):
    run = G.build(w)
    out = G.forward(run)
    rt = G.check_routing(run, out)
    rng = np.random.default_rng(11)
    tokens = np.unique(np.concatenate([np.arange(64), np.arange(w.S - 200, w.S),
                                       rng.choice(w.S, 4096, replace=False)]))
    e_l = G.check_logits(run, out, tokens)
    G.check_losses_own_logits(run, out)
    e_y = G.check_outputs(run, out, rt, tokens[:1024])
    print(f"\n{w.name}: logits rel err {e_l:.2e}, output rel err {e_y:.2e}")
    # a second forward on the same handle gives the same bits
    y1 = out.y.clone()
    out2 = G.forward(run)
    assert torch.equal(out2.y, y1) and np.array_equal(out2.slot, out.slot)
    run.layer.close()
