"""Backward pass, CUDA path vs the oracle (GPU).

The oracle routes the logits the GPU produced (the discrete routing decisions
are held fixed, as in the forward checks) and differentiates in float64.

Comparison: max|got - ref| / max|ref| per gradient, at most 1e-4 for fp32
activations and 2e-2 for bf16 (the forward's output bar), after one allowance:
the ReLU mask [h > 0] is a discontinuous decision taken on a pre-activation
the GPU accumulates in fp32.  Where |pre| is within the fp32 accumulation
bound K * 2^-23 * sum_i |x_i w_i| of zero, either decision is valid, and the
two differ by |x| |dQ| in dW1 and |dQ| |W1| in dx (dQ = dY W2^T, the gradient
before the mask).  The oracle-side slack for those ambiguous elements is
subtracted before the comparison.  dW2, dWg and dbias are continuous in h and
get no allowance.

That bound is loose (it assumes every addition loses a full unit), so each
gradient is also held to a global bar with no allowance at all: the Frobenius
relative error ||got - ref|| / ||ref|| at most 1e-2 (bf16) / 1e-3 (fp32).  A
rounding-decided mask flip moves one rank-one term of one expert, a small part
of the whole norm, while a wrong term anywhere moves it by order one.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from gshard_top_gating_b200 import _lib as L
from gshard_top_gating_b200.inputs import WORKLOADS, Workload, expert_weights, upstream_grad
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
TOL_FRO = {"f32": 1e-3, "bf16": 1e-2}


def _np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _excess_err(got, ref, slack=None) -> float:
    d = np.abs(np.asarray(got, np.float64) - ref)
    if slack is not None:
        d = np.maximum(d - slack, 0.0)
    den = np.abs(ref).max() if ref.size else 0.0
    return float(d.max() / den) if den > 0 else float(d.max() if d.size else 0.0)


def _fro_err(got, ref) -> float:
    den = np.linalg.norm(ref)
    num = np.linalg.norm(np.asarray(got, np.float64) - ref)
    return float(num / den) if den > 0 else float(num)


def _check_all(errs, act):
    for name, e in errs.items():
        bar = TOL_FRO[act] if name.startswith("fro ") else TOL[act]
        assert e <= bar, (name, e)


def _mask_slack(ref, W1, W2, K):
    """Oracle-side bound on what an ambiguous ReLU decision can change."""
    fwd = ref.fwd
    E = W1.shape[0]
    S, M = ref.dx.shape
    s_dW1 = np.zeros_like(ref.dW1)
    s_dxe = np.zeros_like(fwd.xbuf)
    for e in range(E):
        n = int(fwd.n[e])
        if not n:
            continue
        xr = fwd.xbuf[e, :n]
        bound = K * 2.0 ** -23 * (np.abs(xr) @ np.abs(W1[e]))
        amb = np.abs(fwd.hpre[e, :n]) <= bound
        if not amb.any():
            continue
        dq = np.abs(ref.dybuf[e, :n] @ W2[e].T) * amb
        s_dW1[e] = np.abs(xr).T @ dq
        s_dxe[e, :n] = dq @ np.abs(W1[e]).T
    s_dx = np.zeros((S, M))
    for r in range(fwd.slot.shape[1]):
        keep = fwd.slot[:, r] >= 0
        s_dx[keep] += s_dxe[fwd.dest[keep, r], fwd.slot[keep, r]]
    return s_dW1, s_dx


def backward_check(w, a_aux=0.7, a_z=0.3, S=None, train=True, rerouting=False):
    """train: the backward is enabled before the forward, so FFN1 stores the
    ReLU mask bits that dP reads; otherwise dP re-reads h.  rerouting: the
    forward gives dropped choices their second chance (MOE_ROUTE_REROUTE)."""
    run = G.build(w, S=S)
    if train:
        run.layer.enable_backward()
    if rerouting:
        run.layer.set_rerouting(True)
    out = G.forward(run)
    if rerouting:
        rt = O.route(out.logits, w.k, w.cf, rerouting=True)
        assert np.array_equal(out.slot, rt.slot) and (rt.dest != rt.ids).any()
        assert np.array_equal(run.layer.serving_experts(run.S).cpu().numpy(), rt.dest)
    else:
        G.check_routing(run, out)
    dy = upstream_grad(w, device="cuda", S=run.S)
    g = run.layer.backward(out.x, dy, a_aux, a_z)
    torch.cuda.synchronize()
    L.moe_check(run.layer.h)
    W1, W2 = _np(run.W1), _np(run.W2)
    ref = O.backward(_np(out.x), _np(run.Wg), None if run.b is None else _np(run.b), W1, W2, w.k,
                     w.cf, _np(dy), a_aux, a_z, logits=out.logits, rerouting=rerouting)
    s_dW1, s_dx = _mask_slack(ref, W1, W2, w.M)
    errs = {
        "dx": _excess_err(_np(g["dx"]), ref.dx, s_dx),
        "dW1": _excess_err(_np(g["dW1"]), ref.dW1, s_dW1),
        "dW2": _excess_err(_np(g["dW2"]), ref.dW2),
        "dWg": _excess_err(_np(g["dWg"]), ref.dWg),
    }
    for name, r in (("dx", ref.dx), ("dW1", ref.dW1), ("dW2", ref.dW2), ("dWg", ref.dWg)):
        errs["fro " + name] = _fro_err(_np(g[name]), r)
    if run.b is not None:
        errs["dbias"] = _excess_err(_np(g["dbias"]), ref.dbias)
    else:
        assert g["dbias"] is None
    # experts that kept nothing get exactly zero weight gradients
    empty = np.nonzero(ref.fwd.n == 0)[0]
    for e in empty:
        assert not g["dW1"][e].any() and not g["dW2"][e].any()
    return run, out, g, ref, errs


def test_f32_tiny_backward():
    w = WORKLOADS["tiny"]
    run, out, g, ref, errs = backward_check(w)
    print(f"\ntiny f32 backward errors: {errs}")
    _check_all(errs, "f32")
    run.layer.close()


def test_f32_backward_without_loss_terms():
    w = WORKLOADS["tiny"].with_(S=200, cf=0.75)
    run, out, g, ref, errs = backward_check(w, a_aux=0.0, a_z=0.0)
    assert (out.slot < 0).any()
    _check_all(errs, "f32")
    run.layer.close()


BF16_SHAPES = [
    # (S, M, H, E, k, cf, skew_bias)
    (600, 256, 512, 4, 2, 0.5, False),      # a third of the assignments dropped; 256-wide tiles
    (1000, 256, 256, 8, 1, 1.0, False),     # top-1
    (333, 128, 256, 16, 3, 1.0, False),     # ragged kept counts, k = 3
    (257, 192, 320, 6, 2, 1.25, False),     # M, H = 64 mod 128: half-filled last weight-grad tiles
    (512, 128, 128, 64, 2, 1.0, True),      # gate bias: many experts keep nothing (zero tiles)
    (256, 256, 256, 32, 8, 1.25, False),    # top-8
    # experts at capacity (S k / E >= C): the CTA-pair kernels run where 256 divides N or Q
    (768, 384, 256, 4, 2, 1.0, False),      # pair dP and dW1 (P = 384: half-filled last pair tile)
    (1024, 256, 256, 16, 2, 1.0, True),     # pair kernels with experts that keep nothing
    (4096, 512, 1024, 8, 2, 1.0, False),    # several 256-row pair tiles per expert
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=[str(s) for s in BF16_SHAPES])
def test_bf16_backward(shape):
    S, M, H, E, k, cf, skew = shape
    w = Workload("bwd", S, M, H, E, k, cf, "bf16", skew_bias=skew, seed=31)
    run, out, g, ref, errs = backward_check(w)
    print(f"\n{shape}: {errs}")
    _check_all(errs, "bf16")
    run.layer.close()


@pytest.mark.parametrize("shape", [(700, 256, 256, 8, 2, 1.0), (4096, 512, 1024, 8, 2, 1.0)],
                         ids=["one-cta", "cta-pair"])
def test_mask_bits_equal_mask_from_h(shape):
    """dP's ReLU mask from the bits FFN1 stores in training mode and from
    re-reading h select the same elements: all gradients are bitwise equal.
    The second shape puts every expert at capacity (CTA-pair kernels)."""
    S, M, H, E, k, cf = shape
    w = Workload("bits", S, M, H, E, k, cf, "bf16", seed=34)
    run = G.build(w)
    dy = upstream_grad(w, device="cuda")
    run.layer(run.x)                               # forward before the backward is enabled
    g_h = run.layer.backward(run.x, dy, 0.5, 0.1)  # dP re-reads h
    run.layer(run.x)                               # forward in training mode: mask bits
    g_bits = run.layer.backward(run.x, dy, 0.5, 0.1)
    torch.cuda.synchronize()
    for key in g_h:
        if g_h[key] is None:                       # dbias without a gate bias
            assert g_bits[key] is None, key
            continue
        assert torch.equal(g_h[key], g_bits[key]), key
    run.layer.close()


def test_graph_captured_before_training_mode_never_uses_stale_mask_bits():
    """A forward captured in a CUDA graph before the backward is enabled stores no
    mask bits, and the host cannot see its replays.  After a training-mode forward of
    other tokens (which stores bits), a replay of that graph followed by a backward
    must give the replayed forward's gradients: the same as an eager forward and
    backward of the replayed tokens."""
    w = Workload("gbits", 512, 256, 512, 8, 2, 1.25, "bf16", seed=38)
    run = G.build(w)
    dy = upstream_grad(w, device="cuda")
    x = run.x.clone()
    y = torch.empty_like(x)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run.layer(x, out=y)                        # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run.layer(x, out=y)                        # inference epilogue: no mask bits
    run.layer.enable_backward()
    run.layer(torch.roll(run.x, shifts=77, dims=0).contiguous())   # stores bits of other tokens
    x.copy_(torch.flip(run.x, dims=[0]))
    graph.replay()
    g_replay = run.layer.backward(x, dy, 0.5, 0.1)
    torch.cuda.synchronize()
    x_eager = x.clone()
    run.layer(x_eager)
    g_eager = run.layer.backward(x_eager, dy, 0.5, 0.1)
    torch.cuda.synchronize()
    for key in g_eager:
        if g_eager[key] is None:
            continue
        assert torch.equal(g_replay[key], g_eager[key]), key
    del graph
    run.layer.close()


def test_backward_is_deterministic_and_repeatable():
    w = Workload("det", 700, 256, 256, 8, 2, 1.0, "bf16", skew_bias=True, seed=32)
    run = G.build(w)
    x = run.x
    y = run.layer(x)
    dy = upstream_grad(w, device="cuda")
    g1 = run.layer.backward(x, dy, 0.5, 0.1)
    g2 = run.layer.backward(x, dy, 0.5, 0.1)      # a second backward of the same forward
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key
    run.layer(x)                                   # a fresh forward, then again
    g3 = run.layer.backward(x, dy, 0.5, 0.1)
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g3[key]), key
    run.layer.close()


def test_backward_call_order_is_checked():
    w = Workload("order", 128, 128, 128, 4, 2, 1.0, "bf16", seed=33)
    run = G.build(w)
    dy = upstream_grad(w, device="cuda")
    with pytest.raises(L.MoeError) as ei:             # no forward yet
        run.layer.backward(run.x, dy)
    assert ei.value.status == L.MOE_ERR_STATE
    run.layer(run.x)
    with pytest.raises(L.MoeError) as ei:             # a different token count
        run.layer.backward(run.x[:64].contiguous(), dy[:64].contiguous())
    assert ei.value.status == L.MOE_ERR_STATE
    run.layer.route_from_logits(run.layer.logits(128))
    with pytest.raises(L.MoeError) as ei:             # the buffers no longer hold a forward
        run.layer.backward(run.x, dy)
    assert ei.value.status == L.MOE_ERR_STATE
    run.layer.close()


def test_backward_mid_full_size():
    """The mid workload at full size: every token's logit gradient (so dWg and
    dbias in full), the weight gradients of four experts and dx of sampled
    tokens, each from the oracle's step functions one expert or token at a time."""
    w = WORKLOADS["mid"]
    run = G.build(w)
    run.layer.enable_backward()                    # training mode: FFN1 stores the mask bits
    out = G.forward(run)
    rt = G.check_routing(run, out)
    dy = upstream_grad(w, device="cuda")
    a_aux, a_z = 0.01, 0.001
    g = run.layer.backward(out.x, dy, a_aux, a_z)
    torch.cuda.synchronize()
    x = _np(out.x)
    dyn = _np(dy)
    Wg = _np(run.Wg)
    S, E, k = w.S, w.E, w.k
    dgate = np.zeros((S, k))
    rng = np.random.default_rng(7)
    sample_e = set(rng.choice(E, 4, replace=False).tolist())
    tokens = np.unique(np.concatenate([[0, S - 1], rng.choice(S, 256, replace=False)]))
    dxe_rows = {}
    errs = {}
    for e in range(E):
        sel = [(t, r) for r in range(k) for t in np.nonzero((rt.ids[:, r] == e) & (rt.slot[:, r] >= 0))[0]]
        if not sel:
            continue
        sel.sort(key=lambda tr: rt.slot[tr[0], tr[1]])
        ts = np.array([t for t, _ in sel])
        rs = np.array([r for _, r in sel])
        W1e, W2e = (_np(t) for t in expert_weights(w, e))
        xr = x[ts]
        hpre = xr @ W1e
        ye = O.expert_ffn(xr, W1e, W2e)
        dgate[ts, rs] = np.sum(dyn[ts] * ye, axis=1)
        dY = rt.gates[ts, rs][:, None] * dyn[ts]
        want = np.isin(ts, tokens)
        if e in sample_e or want.any():
            dxe, dW1e, dW2e = O.expert_ffn_backward(xr, hpre, dY, W1e, W2e)
            amb = np.abs(hpre) <= w.M * 2.0 ** -23 * (np.abs(xr) @ np.abs(W1e))
            dq = np.abs(dY @ W2e.T) * amb
            for i in np.nonzero(want)[0]:
                dxe_rows[(ts[i], rs[i])] = (dxe[i], dq[i] @ np.abs(W1e).T)
            if e in sample_e:
                errs[f"dW1[{e}]"] = _excess_err(_np(g["dW1"][e]), dW1e, np.abs(xr).T @ dq)
                errs[f"dW2[{e}]"] = _excess_err(_np(g["dW2"][e]), dW2e)
                errs[f"fro dW1[{e}]"] = _fro_err(_np(g["dW1"][e]), dW1e)
                errs[f"fro dW2[{e}]"] = _fro_err(_np(g["dW2"][e]), dW2e)
    dl = O.gates_backward(rt.gates, rt.ids, dgate, E)
    dl += a_aux * O.aux_loss_backward(rt.p, rt.f, E)
    dl += a_z * O.z_loss_backward(rt.p, rt.lse)
    errs["dWg"] = _excess_err(_np(g["dWg"]), x.T @ dl)
    errs["fro dWg"] = _fro_err(_np(g["dWg"]), x.T @ dl)
    errs["dbias"] = _excess_err(_np(g["dbias"]), dl.sum(axis=0)) if g["dbias"] is not None else 0.0
    ref_dx = dl[tokens] @ Wg.T
    slack = np.zeros_like(ref_dx)
    for i, t in enumerate(tokens):
        for r in range(k):
            if (t, r) in dxe_rows:
                ref_dx[i] += dxe_rows[(t, r)][0]
                slack[i] += dxe_rows[(t, r)][1]
    errs["dx"] = _excess_err(_np(g["dx"])[tokens], ref_dx, slack)
    errs["fro dx"] = _fro_err(_np(g["dx"])[tokens], ref_dx)
    print(f"\nmid backward errors: {errs}")
    _check_all(errs, "bf16")
    run.layer.close()


@pytest.mark.parametrize("act,shape", [
    ("bf16", (512, 128, 256, 64, 2, 1.25)),         # one-CTA weight-gradient kernels
    ("bf16", (1024, 256, 256, 16, 2, 1.0)),         # CTA-pair weight-gradient kernels
    ("f32", (256, 64, 128, 32, 2, 1.0)),            # FFMA weight gradients
])
def test_skip_empty_experts_leaves_their_gradients(act, shape):
    """MOE_BWD_SKIP_EMPTY_EXPERTS: experts that kept no token keep the caller's
    bytes; every other gradient equals the dense backward bit for bit."""
    S, M, H, E, k, cf = shape
    w = Workload("skip", S, M, H, E, k, cf, act, skew_bias=True, seed=34)
    run = G.build(w)
    x = run.x
    run.layer(x)
    dy = upstream_grad(w, device="cuda")
    dense = run.layer.backward(x, dy, 0.5, 0.1)
    sentinel = {"dW1": torch.full_like(dense["dW1"], 7.0), "dW2": torch.full_like(dense["dW2"], -3.0)}
    sparse = run.layer.backward(x, dy, 0.5, 0.1, out=sentinel, skip_empty_experts=True)
    torch.cuda.synchronize()
    _, _, _, cnt = run.layer.routing(S)
    empty = (cnt == 0).cpu()
    assert empty.any() and not empty.all()
    for key, fill in (("dW1", 7.0), ("dW2", -3.0)):
        got, ref = sparse[key].cpu(), dense[key].cpu()
        assert torch.all(got[empty] == fill), key
        assert torch.equal(got[~empty], ref[~empty]), key
    for key in ("dx", "dWg", "dbias"):
        if dense[key] is not None:
            assert torch.equal(sparse[key], dense[key]), key
    run.layer.close()


def test_backward_large_sampled():
    """The large workload at full size (experts at capacity: the CTA-pair backward
    kernels over many tiles and waves): 16 rows of dW2[e] and 16 columns of dW1[e]
    for four experts, and dx of tokens whose kept choices all lie in those experts,
    each from the oracle's step functions (no gate-weight gradient here: it needs
    every kept row's FFN output; the mid test checks it in full)."""
    w = WORKLOADS["large"]
    run = G.build(w)
    run.layer.enable_backward()                    # training mode: FFN1 stores the mask bits
    out = G.forward(run)
    rt = G.check_routing(run, out)
    dy = upstream_grad(w, device="cuda")
    a_aux, a_z = 0.01, 0.001
    g = run.layer.backward(out.x, dy, a_aux, a_z)
    torch.cuda.synchronize()
    S, E, k, M, H = w.S, w.E, w.k, w.M, w.H
    rng = np.random.default_rng(11)
    sample_e = sorted(rng.choice(E, 4, replace=False).tolist())
    errs = {}
    W = {}
    for e in sample_e:
        W[e] = (_np(run.W1[e]), _np(run.W2[e]))
        sel = [(t, r) for r in range(k) for t in np.nonzero((rt.ids[:, r] == e) & (rt.slot[:, r] >= 0))[0]]
        sel.sort(key=lambda tr: rt.slot[tr[0], tr[1]])
        ts = np.array([t for t, _ in sel])
        rs = np.array([r for _, r in sel])
        W1e, W2e = W[e]
        xr = _np(out.x[torch.as_tensor(ts, device="cuda")])
        dY = rt.gates[ts, rs][:, None] * _np(dy[torch.as_tensor(ts, device="cuda")])
        cols = rng.choice(H, 16, replace=False)
        # dW2[e][cols, :] = relu(pre[:, cols])^T dY
        pre_c = xr @ W1e[:, cols]
        ref2 = np.maximum(pre_c, 0.0).T @ dY
        got2 = _np(g["dW2"][e])[cols]
        errs[f"dW2[{e}] rows"] = _excess_err(got2, ref2)
        errs[f"fro dW2[{e}] rows"] = _fro_err(got2, ref2)
        # dW1[e][:, cols] = X^T ((dY W2[e][cols]^T) * [pre[:, cols] > 0])
        dq = dY @ W2e[cols].T
        amb = np.abs(pre_c) <= M * 2.0 ** -23 * (np.abs(xr) @ np.abs(W1e[:, cols]))
        ref1 = xr.T @ (dq * (pre_c > 0))
        slack1 = np.abs(xr).T @ (np.abs(dq) * amb)
        got1 = _np(g["dW1"][e])[:, cols]
        errs[f"dW1[{e}] cols"] = _excess_err(got1, ref1, slack1)
        errs[f"fro dW1[{e}] cols"] = _fro_err(got1, ref1)
    # dx of tokens whose kept choices all lie in the sampled experts
    kept = rt.slot >= 0
    inset = np.isin(rt.ids, sample_e) | ~kept
    toks = np.nonzero(inset.all(axis=1) & kept.any(axis=1))[0][:48]
    assert len(toks) >= 8
    xs = _np(out.x[torch.as_tensor(toks, device="cuda")])
    dys = _np(dy[torch.as_tensor(toks, device="cuda")])
    Wg = _np(run.Wg)
    dgate = np.zeros((len(toks), k))
    dxe = np.zeros((len(toks), M))
    slack = np.zeros((len(toks), M))
    for i, t in enumerate(toks):
        for r in range(k):
            if rt.slot[t, r] < 0:
                continue
            W1e, W2e = W[int(rt.ids[t, r])]
            pre = xs[i] @ W1e
            yrow = np.maximum(pre, 0.0) @ W2e
            dgate[i, r] = dys[i] @ yrow
            dq = (rt.gates[t, r] * dys[i]) @ W2e.T
            amb = np.abs(pre) <= M * 2.0 ** -23 * (np.abs(xs[i]) @ np.abs(W1e))
            dxe[i] += (dq * (pre > 0)) @ W1e.T
            slack[i] += (np.abs(dq) * amb) @ np.abs(W1e).T
    dl = O.gates_backward(rt.gates[toks], rt.ids[toks], dgate, E)
    dl += a_aux * O.aux_loss_backward(rt.p[toks], rt.f, E, S=S)
    dl += a_z * O.z_loss_backward(rt.p[toks], rt.lse[toks], S=S)
    ref_dx = dxe + dl @ Wg.T
    got_dx = _np(g["dx"][torch.as_tensor(toks, device="cuda")])
    errs["dx"] = _excess_err(got_dx, ref_dx, slack)
    errs["fro dx"] = _fro_err(got_dx, ref_dx)
    print(f"\nlarge backward errors ({len(toks)} tokens): {errs}")
    _check_all(errs, "bf16")
    run.layer.close()
    del run
    torch.cuda.empty_cache()


def test_backward_wide_sampled():
    """The wide workload at full size (top-8 of 256 experts, 7168-wide rows, one-CTA
    backward kernels): 16 rows of dW2[e] and 16 columns of dW1[e] for four experts, and
    dx of eight tokens with all their kept choices (up to 64 experts), each from the
    oracle's step functions one expert at a time."""
    w = WORKLOADS["wide"]
    run = G.build(w)
    run.layer.enable_backward()
    out = G.forward(run)
    rt = G.check_routing(run, out)
    dy = upstream_grad(w, device="cuda")
    a_aux, a_z = 0.01, 0.001
    g = run.layer.backward(out.x, dy, a_aux, a_z)
    torch.cuda.synchronize()
    S, E, k, M, H = w.S, w.E, w.k, w.M, w.H
    rng = np.random.default_rng(13)
    toks = np.sort(rng.choice(S, 8, replace=False))
    used = sorted(set(int(e) for t in toks for r in range(k) if rt.slot[t, r] >= 0 for e in [rt.ids[t, r]]))
    sample_e = sorted(rng.choice(used, 4, replace=False).tolist())
    xs = _np(out.x[torch.as_tensor(toks, device="cuda")])
    dys = _np(dy[torch.as_tensor(toks, device="cuda")])
    dgate = np.zeros((len(toks), k))
    dxe = np.zeros((len(toks), M))
    slack = np.zeros((len(toks), M))
    errs = {}
    for e in used:
        W1e, W2e = _np(run.W1[e]), _np(run.W2[e])
        for i, t in enumerate(toks):                  # this expert's share of the sampled tokens' dx
            for r in range(k):
                if rt.slot[t, r] < 0 or rt.ids[t, r] != e:
                    continue
                pre = xs[i] @ W1e
                dgate[i, r] = dys[i] @ (np.maximum(pre, 0.0) @ W2e)
                dq = (rt.gates[t, r] * dys[i]) @ W2e.T
                amb = np.abs(pre) <= M * 2.0 ** -23 * (np.abs(xs[i]) @ np.abs(W1e))
                dxe[i] += (dq * (pre > 0)) @ W1e.T
                slack[i] += (np.abs(dq) * amb) @ np.abs(W1e).T
        if e not in sample_e:
            continue
        sel = [(t, r) for r in range(k) for t in np.nonzero((rt.ids[:, r] == e) & (rt.slot[:, r] >= 0))[0]]
        sel.sort(key=lambda tr: rt.slot[tr[0], tr[1]])
        ts = np.array([t for t, _ in sel])
        rs = np.array([r for _, r in sel])
        xr = _np(out.x[torch.as_tensor(ts, device="cuda")])
        dY = rt.gates[ts, rs][:, None] * _np(dy[torch.as_tensor(ts, device="cuda")])
        cols = rng.choice(H, 16, replace=False)
        pre_c = xr @ W1e[:, cols]
        ref2 = np.maximum(pre_c, 0.0).T @ dY
        got2 = _np(g["dW2"][e])[cols]
        errs[f"dW2[{e}] rows"] = _excess_err(got2, ref2)
        errs[f"fro dW2[{e}] rows"] = _fro_err(got2, ref2)
        dq = dY @ W2e[cols].T
        amb = np.abs(pre_c) <= M * 2.0 ** -23 * (np.abs(xr) @ np.abs(W1e[:, cols]))
        ref1 = xr.T @ (dq * (pre_c > 0))
        got1 = _np(g["dW1"][e])[:, cols]
        errs[f"dW1[{e}] cols"] = _excess_err(got1, ref1, np.abs(xr).T @ (np.abs(dq) * amb))
        errs[f"fro dW1[{e}] cols"] = _fro_err(got1, ref1)
    dl = O.gates_backward(rt.gates[toks], rt.ids[toks], dgate, E)
    dl += a_aux * O.aux_loss_backward(rt.p[toks], rt.f, E, S=S)
    dl += a_z * O.z_loss_backward(rt.p[toks], rt.lse[toks], S=S)
    ref_dx = dxe + dl @ _np(run.Wg).T
    got_dx = _np(g["dx"][torch.as_tensor(toks, device="cuda")])
    errs["dx"] = _excess_err(got_dx, ref_dx, slack)
    errs["fro dx"] = _fro_err(got_dx, ref_dx)
    print(f"\nwide backward errors ({len(toks)} tokens over {len(used)} experts): {errs}")
    _check_all(errs, "bf16")
    run.layer.close()
    del run
    torch.cuda.empty_cache()


def test_backward_stage_times():
    """With profiling on, the backward records its eight stages."""
    w = Workload("prof", 512, 256, 256, 8, 2, 1.25, "bf16", seed=35)
    run = G.build(w)
    run.layer(run.x)
    dy = upstream_grad(w, device="cuda")
    run.layer.backward(run.x, dy)                # allocates the backward workspace
    L.moe_set_profiling(run.layer.h, True)
    run.layer(run.x)
    run.layer.backward(run.x, dy)
    ms = L.moe_get_backward_stage_times(run.layer.h)
    L.moe_set_profiling(run.layer.h, False)
    assert len(ms) == L.MOE_NUM_BWD_STAGES and all(t >= 0.0 for t in ms) and sum(ms) > 0.0
    assert [L.moe_backward_stage_name(i) for i in range(len(ms))] == list(L.BWD_STAGES)
    run.layer.close()


EDGE = [
    # (S, M, H, E, k, cf, act, skew_bias)
    (1, 128, 128, 4, 2, 1.0, "bf16", False),      # one token
    (300, 128, 256, 1, 1, 1.0, "bf16", False),    # one expert: a dense FFN, no gate gradient
    (200, 128, 128, 4, 4, 1.0, "bf16", False),    # k = E
    (97, 64, 128, 6, 2, 0.75, "f32", True),       # fp32 with a gate bias and drops
    (65, 64, 64, 3, 3, 2.0, "f32", False),        # fp32, k = E, no drops
]


@pytest.mark.parametrize("shape", EDGE, ids=[str(s) for s in EDGE])
def test_backward_edge_shapes(shape):
    S, M, H, E, k, cf, act, skew = shape
    w = Workload("edge", S, M, H, E, k, cf, act, skew_bias=skew, seed=36)
    # one expert: the gate and l_aux gradients vanish (g = p = 1); with a_z = 0 so does dW_g
    run, out, g, ref, errs = backward_check(w, a_z=0.0 if E == 1 else 0.3)
    print(f"\n{shape}: {errs}")
    _check_all(errs, act)
    if E == 1:
        assert np.abs(_np(g["dWg"])).max() <= 1e-6 * np.abs(_np(g["dx"])).max()
    run.layer.close()


@pytest.mark.parametrize("w", [
    Workload("bwd_rr_bf16", 900, 128, 256, 16, 2, 0.6, "bf16", skew_bias=True),
    Workload("bwd_rr_bf16_k3", 500, 256, 128, 12, 3, 0.5, "bf16", skew_bias=True),
    Workload("bwd_rr_f32", 300, 64, 128, 8, 2, 0.6, "f32", skew_bias=True),
], ids=lambda w: w.name)
def test_backward_of_rerouted_forward(w):
    """Rows of a rerouted choice sit at the serving expert; its gate gradient goes to
    the expert it chose (oracle `backward(..., rerouting=True)`)."""
    run, out, g, ref, errs = backward_check(w, rerouting=True)
    print(f"\n{w.name}: {errs}")
    _check_all(errs, w.act)
    run.layer.close()
