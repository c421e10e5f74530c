"""Shared logic of the GPU parity tests: run the CUDA path, check it against the oracle.

Tolerances (the layer's stated parity bar):
  routing (expert ids, slots, drop mask, per-expert demand): bit-exact, given the
      same fp32 logits -- the oracle routes the logits the GPU produced;
  logits: max|d| / max|ref| <= 1e-5 against the oracle's own float64 product;
  gates: |d| <= 2e-6 |ref| + 1e-9 (device expf vs host exp);
  layer output: max|d| / max|ref| <= 1e-4 (fp32) and <= 2e-2 (bf16);
  l_aux and z: relative 1e-5, both on the GPU's logits and on the oracle's own.
"""
from __future__ import annotations

from types import SimpleNamespace

import numpy as np
import torch

import oracle as O
from gshard_top_gating_b200.inputs import make_inputs
from gshard_top_gating_b200.layer import MoeLayer

TOL_LOGITS = 1e-5
TOL_LOSS = 1e-5
TOL_Y = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max() if ref.size else 0.0
    num = np.abs(got - ref).max() if ref.size else 0.0
    if den == 0.0:
        return float(num)
    return float(num / den)


def build(w, S=None, device="cuda", S_max=None):
    S = w.S if S is None else S
    x, Wg, b, W1, W2 = make_inputs(w, device=device, S=S)
    layer = MoeLayer(S_max or max(S, 1), w.M, w.H, w.E, w.k, w.cf, Wg, b, W1, W2)
    return SimpleNamespace(w=w, S=S, x=x, Wg=Wg, b=b, W1=W1, W2=W2, layer=layer)


def forward(run, S=None):
    S = run.S if S is None else S
    x = run.x[:S].contiguous()
    y = run.layer(x)
    l_aux, z = run.layer.aux_loss()
    torch.cuda.synchronize()
    eidx, gate, slot, cnt = (t.cpu().numpy() for t in run.layer.routing(S))
    return SimpleNamespace(S=S, x=x, y=y, l_aux=l_aux, z=z, logits=run.layer.logits(S).cpu().numpy(),
                           eidx=eidx, gate=gate, slot=slot, cnt=cnt)


def check_routing(run, out):
    """Routing bit-exact and losses given the GPU's logits; returns the oracle's route."""
    w = run.w
    rt = O.route(out.logits, w.k, w.cf)
    assert np.array_equal(out.eidx, rt.ids), "expert ids differ"
    assert np.array_equal(out.slot, rt.slot), "slots / drop mask differ"
    assert np.array_equal(out.cnt, rt.cnt), "per-expert demand differs"
    if out.S:
        assert np.all(np.abs(out.gate - rt.gates) <= 2e-6 * np.abs(rt.gates) + 1e-9), "gates"
        assert abs(out.l_aux - rt.l_aux) <= TOL_LOSS * abs(rt.l_aux), (out.l_aux, rt.l_aux)
        assert abs(out.z - rt.z) <= TOL_LOSS * abs(rt.z), (out.z, rt.z)
    return rt


def check_logits(run, out, tokens):
    xs = run.x[torch.as_tensor(tokens, device=run.x.device)].cpu()
    ref = O.gate_logits(xs, run.Wg.cpu(), None if run.b is None else run.b.cpu())
    err = rel_err(out.logits[tokens], ref)
    assert err <= TOL_LOGITS, err
    return err


def check_losses_own_logits(run, out):
    ref = O.gate_logits(out.x.cpu(), run.Wg.cpu(), None if run.b is None else run.b.cpu())
    rt = O.route(ref, run.w.k, run.w.cf)
    assert abs(out.l_aux - rt.l_aux) <= TOL_LOSS * abs(rt.l_aux), (out.l_aux, rt.l_aux)
    assert abs(out.z - rt.z) <= TOL_LOSS * abs(rt.z), (out.z, rt.z)


def check_outputs(run, out, rt, tokens):
    tokens = np.asarray(tokens, dtype=np.int64)
    xs = run.x[torch.as_tensor(tokens, device=run.x.device)].cpu()
    W1, W2 = run.W1, run.W2
    ref = O.outputs_for_tokens(tokens, xs, rt.ids, rt.gates, rt.slot,
                               lambda e: (W1[e].cpu(), W2[e].cpu()))
    got = out.y[torch.as_tensor(tokens, device=out.y.device)].float().cpu().numpy()
    # tokens whose every choice was dropped are exactly zero
    dropped = np.all(rt.slot[tokens] < 0, axis=1)
    assert np.all(got[dropped] == 0.0)
    err = rel_err(got, ref)
    assert err <= TOL_Y[run.w.act], err
    return err


def full_check(run, S=None):
    out = forward(run, S)
    rt = check_routing(run, out)
    if out.S:
        check_logits(run, out, np.arange(out.S))
        check_outputs(run, out, rt, np.arange(out.S))
        check_losses_own_logits(run, out)
    return out, rt
