"""CPU oracle for the GShard top-2 (top-k) MoE layer, forward and backward.  TEST INFRASTRUCTURE.

This file exists to check the CUDA path, never to serve it.  Only `tests/`,
`__graft_entry__.smoke()` and `bench.py`'s CPU-baseline / reference arm may
import it; the library under `gshard_top_gating_b200/` never does, and it shares
no code, table or helper with it.

Everything is plain numpy in float64 (inputs given in fp32 or bf16 are upcast
exactly).  A library matmul or cumulative sum serves as a step where the
definition is a plain matrix product or count; there is no blocking, fusion or
reordering beyond that.

Sources (the web pages this method is taken from):

[gist]  "GShard (Expert Parallelism)", learn card, "In plain words": experts sit
        in per-device buffers, tokens go out to them and come back; capacity
        factors bound each expert's load.
[note]  "GShard: Scaling Giant Models with Conditional Computation and Automatic
        Sharding", paper note, summary paragraph: top-2 gating with
        softmax-normalised top-2 weights; auxiliary load-balance loss
        N * sum_j f_j * P_j plus a z-loss; tokens beyond an expert's capacity
        (set by capacity_factor) are dropped.
[blog]  "GShard: Scaling Giant Neural Networks with Conditional Computation",
        section "Mixture-of-Experts Implementation": G(x) = Softmax(x . W_g),
        top-k with k = 2 typical, the "Expert Capacity" paragraph; section "Core
        Components", "Expert Networks": each expert is a Transformer-style
        feed-forward network.

Readings where the pages are silent (each one is listed in the design notes):
 * N in N*sum f_j P_j is the number of experts E; f_j is the fraction of tokens
   whose FIRST choice is j, counted before capacity; P_j is the mean over tokens
   of the full softmax probability of expert j.
 * z-loss = mean over tokens of logsumexp(logits)^2, unweighted.
 * The normalised top-k weights are g_r = p_{e_r} / sum_{r'<k} p_{e_r'}.
 * Capacity C = ceil(capacity_factor * k * S / E), evaluated in double.
 * Slots are handed out rank-major: all first choices in token order, then all
   second choices, and so on; an assignment whose expert is full is dropped and
   contributes zero; the surviving weights are not renormalised.
 * Top-k selects on the fp32 logits, ties to the lower expert index.
 * The expert FFN is relu(x W1[e]) W2[e] with no biases.
 * Rerouting (optional, off by default): a dropped assignment is offered once
   to the token's next-ranked unchosen expert, in the capacity pass's order,
   into the capacity left over; it keeps its gate weight (see `reroute`).
 * An empty batch (S = 0) has l_aux = z = 0.
 * Backward: the routing (choices, slots, drops) and the first-choice fractions
   f_j carry no gradient; every other step is differentiated exactly.

Pins: every forward function here is checked in tests/test_oracle_pins.py
against hand examples, closed forms, library routines, brute force and
invariants; the backward in tests/test_oracle_backward_pins.py against central
finite differences of the forward and the textbook dense-FFN backward.
"""
from __future__ import annotations

import math
from types import SimpleNamespace

import numpy as np

__all__ = [
    "capacity", "gate_logits", "softmax_stats", "top_k", "normalized_gates",
    "assign_slots", "reroute", "expert_ffn", "dispatch", "combine", "aux_losses",
    "route", "forward", "expert_ffn_backward", "gates_backward", "aux_loss_backward",
    "z_loss_backward", "backward", "outputs_for_tokens",
]


def _f64(a) -> np.ndarray:
    """Exact upcast of a numpy array or torch tensor (fp32 / bf16 / f64) to float64."""
    if hasattr(a, "detach"):          # torch tensor (bf16 has no numpy dtype)
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def capacity(S: int, E: int, k: int, cf: float) -> int:
    """Expert capacity C = ceil(cf * k * S / E).

    [note] summary: over-capacity tokens are dropped, "governed by
    capacity_factor"; [blog] "Expert Capacity": each expert processes at most a
    fixed number of tokens per batch.  The formula itself is the reading above.
    """
    return int(math.ceil(cf * k * S / E))


def gate_logits(x, Wg, bias=None, round_fp32: bool = True) -> np.ndarray:
    """Gating logits l = x . W_g (+ b), returned as float32 [S, E].

    [blog] "Mixture-of-Experts Implementation", G(x) = Softmax(x . W_g): the
    product is taken in float64 and rounded once to float32; a per-expert bias,
    when given, is added in float32 after that rounding.  With
    round_fp32=False everything stays float64 (for finite-difference checks of
    the backward pass, which fp32 rounding would drown).
    """
    if not round_fp32:
        l = _f64(x) @ _f64(Wg)
        return l if bias is None else l + _f64(bias)
    l = (_f64(x) @ _f64(Wg)).astype(np.float32)
    if bias is not None:
        l = (l + np.asarray(_f64(bias), dtype=np.float32)).astype(np.float32)
    return l


def softmax_stats(logits):
    """Softmax probabilities p[S,E] and log-sum-exp lse[S] of the logits, float64.

    [blog] "Mixture-of-Experts Implementation": G(x) = Softmax(x . W_g).
    """
    l = _f64(logits)
    if l.shape[0] == 0:
        return np.zeros_like(l), np.zeros(0)
    mx = l.max(axis=1, keepdims=True)
    ex = np.exp(l - mx)
    s = ex.sum(axis=1, keepdims=True)
    p = ex / s
    lse = (mx + np.log(s))[:, 0]
    return p, lse


def top_k(logits, k: int) -> np.ndarray:
    """Expert ids [S, k] int32: the k largest logits per token, best first.

    [note] "top-2"; [blog] "top-k experts (typically k=2)".  Selection is on
    the logits (order-equivalent to the probabilities); ties go to the lower
    expert index (np.argmax returns the first maximum).  float64 logits are
    compared as given.
    """
    l = np.array(logits, dtype=np.float64 if np.asarray(logits).dtype == np.float64 else np.float32,
                 copy=True)
    assert np.all(np.isfinite(l)), "logits must be finite"
    S = l.shape[0]
    ids = np.zeros((S, k), dtype=np.int32)
    rows = np.arange(S)
    for r in range(k):
        j = np.argmax(l, axis=1) if S else np.zeros(0, dtype=np.int64)
        ids[:, r] = j
        l[rows, j] = -np.inf
    return ids


def normalized_gates(p, ids) -> np.ndarray:
    """Gate weights g[S, k] = p[t, e_r] / sum_{r'} p[t, e_r'] (float64).

    [note] "softmax-normalised top-2 weights".
    """
    p = _f64(p)
    sel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def assign_slots(ids, E: int, C: int):
    """Capacity-limited slot assignment.

    Returns slot[S, k] int32 (-1 where dropped) and cnt[E] int64 (demand, before
    capacity).  Rank-major order: for r = 0..k-1 and tokens in order, the
    position of (t, r) at expert e is the number of earlier assignments to e;
    it is kept iff that position is below C.  [note] summary (dropping beyond
    capacity), [blog] "Expert Capacity".
    """
    ids = np.asarray(ids)
    S, k = ids.shape
    slot = np.full((S, k), -1, dtype=np.int32)
    cnt = np.zeros(E, dtype=np.int64)
    experts = np.arange(E)
    for r in range(k):
        onehot = (ids[:, r][:, None] == experts[None, :]).astype(np.int64)   # [S, E]
        earlier = np.cumsum(onehot, axis=0) - onehot                            # same-rank, earlier tokens
        pos = cnt[ids[:, r]] + earlier[np.arange(S), ids[:, r]]
        slot[:, r] = np.where(pos < C, pos, -1)
        cnt += onehot.sum(axis=0)
    return slot, cnt


def reroute(logits, ids, slot, cnt, C: int):
    """Second chance for the assignments the capacity pass dropped.

    [blog] "Expert Capacity": tokens over an expert's capacity are either dropped
    or routed to alternative experts; the page gives no rule for the second
    option.  Reading taken here: each dropped assignment (t, r) is offered to one
    alternative expert, the best-ranked expert of token t (largest logit, ties to
    the lower index) that t did not choose and that no earlier dropped
    assignment of t was offered -- the token's j-th dropped assignment (in r
    order) is offered its (k + j)-th ranked expert.  Offers are taken in the
    capacity pass's order (r, then t); an expert accepts while it has free slots
    (C minus the rows the capacity pass kept) and gives the next one.  A rerouted
    assignment keeps its gate weight g_r; one not accepted stays dropped.

    Returns dest[S, k] (the expert that serves each assignment: the chosen one
    unless rerouted), slot[S, k] (-1 if dropped) and n[E] (kept rows per expert).
    """
    l = np.asarray(logits)
    ids = np.asarray(ids)
    S, k = ids.shape
    E = l.shape[1]
    ranking = top_k(l, E)                       # every expert, best first
    n = np.minimum(np.asarray(cnt), C).astype(np.int64)
    dest = ids.astype(np.int32).copy()
    out = np.array(slot, dtype=np.int32, copy=True)
    j = np.zeros((S, k), dtype=np.int64)        # earlier dropped assignments of the token
    for r in range(1, k):
        j[:, r] = j[:, r - 1] + (np.asarray(slot)[:, r - 1] < 0)
    for r in range(k):
        for t in range(S):
            if slot[t, r] >= 0 or k + j[t, r] >= E:
                continue
            a = ranking[t, k + j[t, r]]
            if n[a] < C:
                out[t, r] = n[a]
                dest[t, r] = a
                n[a] += 1
    return dest, out, n


def expert_ffn(rows, W1e, W2e) -> np.ndarray:
    """One expert's two-layer ReLU feed-forward network: relu(rows W1e) W2e.

    [blog] "Core Components", "Expert Networks" (Transformer-style FFN, no
    biases by the reading above).
    """
    h = np.maximum(_f64(rows) @ _f64(W1e), 0.0)
    return h @ _f64(W2e)


def dispatch(x, ids, slot, E: int, C: int) -> np.ndarray:
    """Per-expert capacity buffers xbuf[E, C, M]: xbuf[e_r, slot_r] = x[t] for kept (t, r).

    [gist] "In plain words": tokens are sent to the experts' buffers (on one
    device the all-to-all becomes this permutation).  Unused rows are zero.
    """
    x = _f64(x)
    S, M = x.shape
    xbuf = np.zeros((E, C, M))
    for r in range(ids.shape[1]):
        keep = slot[:, r] >= 0
        xbuf[ids[keep, r], slot[keep, r]] = x[keep]
    return xbuf


def combine(ybuf, ids, gates, slot) -> np.ndarray:
    """Gate-weighted combine y[t] = sum_{r kept} g_r * ybuf[e_r, slot_r].

    [gist] "In plain words" (results are returned to their tokens); the
    weighting by the normalised gates follows [note].  Dropped assignments
    contribute zero and the kept weights are not renormalised.
    """
    S, k = ids.shape
    y = np.zeros((S, ybuf.shape[2]))
    for r in range(k):
        keep = slot[:, r] >= 0
        y[keep] += gates[keep, r][:, None] * ybuf[ids[keep, r], slot[keep, r]]
    return y


def aux_losses(p, ids, lse, E: int):
    """Auxiliary load-balance loss l_aux = E * sum_j f_j P_j and z-loss mean(lse^2).

    [note] summary: "N * sum_j f_j * P_j plus a z-loss" (readings of N, f_j,
    P_j and the z-loss above).  Returns (l_aux, z, f, P) as floats / float64.
    """
    p = _f64(p)
    S = p.shape[0]
    if S == 0:
        return 0.0, 0.0, np.zeros(E), np.zeros(E)
    P = p.sum(axis=0) / S
    f = np.bincount(np.asarray(ids)[:, 0], minlength=E).astype(np.float64) / S
    l_aux = float(E * np.sum(f * P))
    z = float(np.sum(_f64(lse) ** 2) / S)
    return l_aux, z, f, P


def route(logits, k: int, cf: float, rerouting: bool = False):
    """Routing of given fp32 logits: everything between the gate GEMM and dispatch.

    Returns a namespace with p, lse, ids, gates, C, slot, cnt, n, l_aux, z and
    dest (the expert serving each assignment: ids, unless `rerouting` gives a
    dropped assignment a second chance, see `reroute`; then slot and n are the
    final ones and slot0 the capacity pass's).  float64 logits (finite-difference
    checks) are routed without rounding.
    """
    logits = np.asarray(logits)
    if logits.dtype != np.float64:
        logits = logits.astype(np.float32)
    S, E = logits.shape
    C = capacity(S, E, k, cf)
    p, lse = softmax_stats(logits)
    ids = top_k(logits, k)
    g = normalized_gates(p, ids) if S else np.zeros((0, k))
    slot, cnt = assign_slots(ids, E, C)
    l_aux, z, f, P = aux_losses(p, ids, lse, E)
    slot0, dest, n = slot, ids, np.minimum(cnt, C)
    if rerouting:
        dest, slot, n = reroute(logits, ids, slot0, cnt, C)
    return SimpleNamespace(p=p, lse=lse, ids=ids, gates=g, C=C, slot=slot, cnt=cnt,
                           n=n, l_aux=l_aux, z=z, f=f, P=P, dest=dest, slot0=slot0)


def forward(x, Wg, bias, W1, W2, k: int, cf: float, round_fp32: bool = True, logits=None,
            rerouting: bool = False):
    """The whole layer forward on the CPU (small cases).

    Returns the `route` namespace plus logits, the per-expert buffers (xbuf,
    pre-activation hpre, ybuf) and the output y[S, M] (float64).  Given
    `logits` (fp32 [S, E], bias included) the routing uses them instead of
    x . W_g + b, so that a check can hold the discrete routing decisions fixed.
    With `rerouting`, dropped assignments get their second chance (`reroute`)
    and are dispatched to and combined from the expert that serves them.
    """
    if logits is None:
        logits = gate_logits(x, Wg, bias, round_fp32)
    rt = route(logits, k, cf, rerouting)
    S, E = logits.shape
    C = rt.C
    W1 = _f64(W1)
    W2 = _f64(W2)
    xbuf = dispatch(x, rt.dest, rt.slot, E, C)
    ybuf = np.zeros_like(xbuf)
    hpre = np.zeros((E, C, W1.shape[2]))
    for e in range(E):
        n = int(rt.n[e])
        if n:
            ybuf[e, :n] = expert_ffn(xbuf[e, :n], W1[e], W2[e])
            hpre[e, :n] = xbuf[e, :n] @ W1[e]
    rt.logits = logits
    rt.xbuf, rt.hpre, rt.ybuf = xbuf, hpre, ybuf
    rt.y = combine(ybuf, rt.dest, rt.gates, rt.slot)
    return rt


def expert_ffn_backward(rows, hpre, dY, W1e, W2e):
    """Backward of one expert's ReLU FFN y = relu(rows W1e) W2e ([blog] Expert Networks).

    Given the upstream gradient dY of the expert's outputs: dW2 = relu(pre)^T dY,
    dpre = (dY W2^T) * [pre > 0], dW1 = rows^T dpre, drows = dpre W1^T.
    Returns (drows, dW1e, dW2e).
    """
    h = np.maximum(hpre, 0.0)
    dW2e = h.T @ dY
    dpre = (dY @ W2e.T) * (hpre > 0)
    return dpre @ W1e.T, rows.T @ dpre, dW2e


def gates_backward(gates, ids, dgate, E: int):
    """Logit gradient through the normalised gates g_r = softmax over the k chosen logits.

    [note] "softmax-normalised top-2 weights": dl[t, e_r] += g_r (dgate_r -
    sum_r' g_r' dgate_r').  Returns dl[S, E].
    """
    S, k = gates.shape
    dl = np.zeros((S, E))
    inner = np.sum(gates * dgate, axis=1, keepdims=True)
    np.add.at(dl, (np.arange(S)[:, None].repeat(k, 1), ids), gates * (dgate - inner))
    return dl


def aux_loss_backward(p, f, E: int, S: int | None = None):
    """d l_aux / d logits with f_j held fixed (a count of argmax choices carries no gradient).

    l_aux = E sum_j f_j P_j, P_j = mean_t p[t, j]; through the softmax:
    dl[t] = E/S * p_t * (f - <p_t, f>).  Returns dl for the rows of p; S is the
    batch's token count (default: the rows given).
    """
    S = p.shape[0] if S is None else S
    return E / S * p * (f[None, :] - (p @ f)[:, None])


def z_loss_backward(p, lse, S: int | None = None):
    """d z / d logits for z = mean_t lse_t^2: dl[t] = 2/S * lse_t * p_t (S as above)."""
    S = p.shape[0] if S is None else S
    return 2.0 / S * lse[:, None] * p


def backward(x, Wg, bias, W1, W2, k: int, cf: float, dy, a_aux: float = 0.0, a_z: float = 0.0,
             round_fp32: bool = True, logits=None, rerouting: bool = False):
    """Gradients of  L = <dy, y> + a_aux * l_aux + a_z * z  with respect to x, W_g, b, W1, W2.

    The routing (expert choice, slots, drops) is piecewise constant and carries
    no gradient; everything else is differentiated exactly, in the forward's
    order reversed:
      combine: dY_e[slot_r] = g_r dy[t] and dgate_r = <dy[t], y_e[slot_r]>
        (both 0 for a dropped assignment);
      expert FFN: `expert_ffn_backward` per expert, dx[t] += sum of the kept
        choices' row gradients;
      gates, l_aux, z: `gates_backward`, `aux_loss_backward`, `z_loss_backward`
        give the logit gradient dl;
      gate GEMM ([blog] G(x) = Softmax(x . W_g)): dx += dl W_g^T, dW_g = x^T dl, db = sum_t dl.
    Returns a namespace with dx, dWg, dbias, dW1, dW2 (float64), the
    intermediates dl, dgate, dybuf (the expert outputs' gradient) and the
    forward namespace fwd.  `logits` as in `forward`.  With `rerouting`, a
    rerouted assignment's rows live at the expert that serves it (dest), while
    its gate weight -- and so its gradient -- belongs to the expert it chose.
    """
    rt = forward(x, Wg, bias, W1, W2, k, cf, round_fp32, logits, rerouting)
    xf, Wgf, W1f, W2f, dyf = _f64(x), _f64(Wg), _f64(W1), _f64(W2), _f64(dy)
    S, E = rt.logits.shape
    dgate = np.zeros((S, k))
    dybuf = np.zeros_like(rt.ybuf)
    for r in range(k):
        keep = rt.slot[:, r] >= 0
        t = np.nonzero(keep)[0]
        e, sl = rt.dest[keep, r], rt.slot[keep, r]
        dgate[t, r] = np.sum(dyf[t] * rt.ybuf[e, sl], axis=1)
        dybuf[e, sl] = rt.gates[t, r][:, None] * dyf[t]
    dW1 = np.zeros_like(W1f)
    dW2 = np.zeros_like(W2f)
    dxbuf = np.zeros_like(rt.xbuf)
    for e in range(E):
        n = int(rt.n[e])
        if n:
            dxbuf[e, :n], dW1[e], dW2[e] = expert_ffn_backward(
                rt.xbuf[e, :n], rt.hpre[e, :n], dybuf[e, :n], W1f[e], W2f[e])
    dx = np.zeros_like(xf)
    for r in range(k):
        keep = rt.slot[:, r] >= 0
        dx[keep] += dxbuf[rt.dest[keep, r], rt.slot[keep, r]]
    dl = np.zeros((S, E))
    if S:
        dl += gates_backward(rt.gates, rt.ids, dgate, E)
        dl += a_aux * aux_loss_backward(rt.p, rt.f, E)
        dl += a_z * z_loss_backward(rt.p, rt.lse)
    dx += dl @ Wgf.T
    dWg = xf.T @ dl
    dbias = dl.sum(axis=0)
    return SimpleNamespace(dx=dx, dWg=dWg, dbias=dbias, dW1=dW1, dW2=dW2, dl=dl, dgate=dgate,
                           dybuf=dybuf, fwd=rt)


def outputs_for_tokens(tokens, x_rows, ids, gates, slot, expert_weights):
    """Layer outputs y[tokens] for a sample of tokens, given the full routing.

    Because xbuf[e_r, slot_r] holds x[t] itself, y[t] = sum_{r kept} g_r *
    FFN_{e_r}(x[t]) depends only on x[t] and the routing of t.  `x_rows[i]` is
    x[tokens[i]]; `expert_weights(e)` returns (W1[e], W2[e]).  Experts are
    visited one at a time so only one expert's weights are held.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    xr = _f64(x_rows)
    y = np.zeros((len(tokens), xr.shape[1]))
    sid = ids[tokens]
    sg = _f64(gates)[tokens]
    ss = slot[tokens]
    for e in np.unique(sid[ss >= 0]):
        W1e, W2e = expert_weights(int(e))
        for r in range(ids.shape[1]):
            sel = np.nonzero((sid[:, r] == e) & (ss[:, r] >= 0))[0]
            if len(sel):
                y[sel] += sg[sel, r][:, None] * expert_ffn(xr[sel], W1e, W2e)
    return y
