"""Pins of the oracle's backward pass (CPU): central finite differences of
L = <dy, y> + a_aux * l_aux + a_z * z computed by the oracle's own forward in
float64, at random coordinates of every input; the routing is held fixed by
choosing cases without near-ties, so the difference quotient sees the smooth
part only.  Planted mistakes in a copy of the backward must be caught too.
"""
import numpy as np
import pytest

import oracle.moe_oracle as M

EPS = 1e-6


def _loss(x, Wg, b, W1, W2, k, cf, dy, a_aux, a_z, rerouting=False):
    rt = M.forward(x, Wg, b, W1, W2, k, cf, round_fp32=False, rerouting=rerouting)
    return float(np.sum(dy * rt.y) + a_aux * rt.l_aux + a_z * rt.z)


def _case(seed, S, Md, H, E, k, cf, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, Md))
    Wg = rng.standard_normal((Md, E))
    b = rng.standard_normal(E) if bias else None
    W1 = rng.standard_normal((E, Md, H)) / np.sqrt(Md)
    W2 = rng.standard_normal((E, H, Md)) / np.sqrt(H)
    dy = rng.standard_normal((S, Md))
    return x, Wg, b, W1, W2, k, cf, dy


def _fd_check(args, a_aux, a_z, grads, n_coords=6, seed=0, rerouting=False):
    x, Wg, b, W1, W2, k, cf, dy = args
    rng = np.random.default_rng(seed)
    names = [("x", x, grads.dx), ("Wg", Wg, grads.dWg), ("W1", W1, grads.dW1), ("W2", W2, grads.dW2)]
    if b is not None:
        names.append(("b", b, grads.dbias))
    for name, arr, g in names:
        for _ in range(n_coords):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            orig = arr[idx]
            arr[idx] = orig + EPS
            lp = _loss(x, Wg, b, W1, W2, k, cf, dy, a_aux, a_z, rerouting)
            arr[idx] = orig - EPS
            lm = _loss(x, Wg, b, W1, W2, k, cf, dy, a_aux, a_z, rerouting)
            arr[idx] = orig
            fd = (lp - lm) / (2 * EPS)
            assert abs(fd - g[idx]) <= 2e-6 + 2e-6 * abs(fd), (name, idx, fd, g[idx])


@pytest.mark.parametrize("seed,S,Md,H,E,k,cf", [
    (1, 10, 6, 5, 4, 2, 0.75),     # some assignments dropped
    (2, 12, 4, 7, 6, 3, 2.0),      # no drops, k = 3
    (3, 9, 5, 4, 3, 1, 1.0),       # top-1
    (4, 8, 4, 6, 5, 5, 1.0),       # k = E
])
def test_backward_matches_finite_differences(seed, S, Md, H, E, k, cf):
    args = _case(seed, S, Md, H, E, k, cf)
    x, Wg, b, W1, W2, k, cf, dy = args
    for a_aux, a_z in ((0.0, 0.0), (0.7, 0.3)):
        grads = M.backward(x, Wg, b, W1, W2, k, cf, dy, a_aux, a_z, round_fp32=False)
        _fd_check(args, a_aux, a_z, grads, seed=seed)


@pytest.mark.parametrize("seed,S,Md,H,E,k,cf", [
    (11, 12, 5, 6, 5, 2, 0.6),      # dropped choices rerouted, some for good
    (12, 10, 4, 5, 6, 3, 0.5),      # k = 3: tokens with two dropped choices
])
def test_rerouted_backward_matches_finite_differences(seed, S, Md, H, E, k, cf):
    """With rerouting, rows live at the serving expert and gates at the chosen one."""
    args = _case(seed, S, Md, H, E, k, cf)
    x, Wg, b, W1, W2, k, cf, dy = args
    rt = M.forward(x, Wg, b, W1, W2, k, cf, round_fp32=False, rerouting=True)
    assert (rt.dest != rt.ids).any(), "the case reroutes something"
    for a_aux, a_z in ((0.0, 0.0), (0.7, 0.3)):
        grads = M.backward(x, Wg, b, W1, W2, k, cf, dy, a_aux, a_z, round_fp32=False, rerouting=True)
        _fd_check(args, a_aux, a_z, grads, seed=seed, rerouting=True)


def test_single_expert_backward_is_dense_ffn_backward():
    # E = 1, k = 1: gate is 1, l_aux = 1 constant; y = relu(x W1) W2
    args = _case(5, 7, 4, 6, 1, 1, 1.0, bias=False)
    x, Wg, _, W1, W2, k, cf, dy = args
    g = M.backward(x, Wg, None, W1, W2, 1, 1.0, dy, a_aux=0.5, a_z=0.0, round_fp32=False)
    pre = x @ W1[0]
    h = np.maximum(pre, 0)
    dpre = (dy @ W2[0].T) * (pre > 0)
    assert np.allclose(g.dW2[0], h.T @ dy, atol=1e-12)
    assert np.allclose(g.dW1[0], x.T @ dpre, atol=1e-12)
    assert np.allclose(g.dx, dpre @ W1[0].T, atol=1e-12)          # no gate / aux gradient
    assert np.allclose(g.dWg, 0.0, atol=1e-12)


def test_dropped_assignments_carry_no_expert_gradient():
    args = _case(6, 16, 4, 5, 2, 2, 0.25)          # C = 4 of 16 per expert
    x, Wg, b, W1, W2, k, cf, dy = args
    g = M.backward(x, Wg, b, W1, W2, k, cf, dy)
    fully = np.all(g.fwd.slot < 0, axis=1)
    assert fully.any()
    assert np.allclose(g.dgate[fully], 0.0)
    # a fully dropped token gets gradient only through the gate GEMM, and with
    # dgate = 0 and no loss weights that is zero too
    assert np.allclose(g.dx[fully], 0.0)


def _no_relu_mask(rows, hpre, dY, W1e, W2e):
    h = np.maximum(hpre, 0.0)
    dpre = dY @ W2e.T                                   # mask forgotten
    return dpre @ W1e.T, rows.T @ dpre, h.T @ dY


def _dw2_without_relu(rows, hpre, dY, W1e, W2e):
    dpre = (dY @ W2e.T) * (hpre > 0)
    return dpre @ W1e.T, rows.T @ dpre, hpre.T @ dY      # pre-activation instead of h


def _gates_uncentred(gates, ids, dgate, E):
    S, k = gates.shape
    dl = np.zeros((S, E))
    np.add.at(dl, (np.arange(S)[:, None].repeat(k, 1), ids), gates * dgate)
    return dl


def _aux_uncentred(p, f, E, S=None):
    return E / (p.shape[0] if S is None else S) * p * f[None, :]


def _z_wrong_sign(p, lse, S=None):
    return -2.0 / (p.shape[0] if S is None else S) * lse[:, None] * p


PLANTS = {
    "expert_ffn_backward": [_no_relu_mask, _dw2_without_relu],
    "gates_backward": [_gates_uncentred],
    "aux_loss_backward": [_aux_uncentred],
    "z_loss_backward": [_z_wrong_sign],
}


@pytest.mark.parametrize("name,bad", [(n, f) for n, fs in PLANTS.items() for f in fs],
                         ids=[f.__name__ for fs in PLANTS.values() for f in fs])
def test_finite_differences_catch_planted_mistakes(monkeypatch, name, bad):
    """Each mistake is planted in the oracle's own step function; the pins must fail."""
    args = _case(7, 10, 5, 6, 4, 2, 1.0)
    x, Wg, b, W1, W2, k, cf, dy = args
    good = M.backward(x, Wg, b, W1, W2, k, cf, dy, 0.7, 0.3, round_fp32=False)
    _fd_check(args, 0.7, 0.3, good, seed=7)
    monkeypatch.setattr(M, name, bad)
    planted = M.backward(x, Wg, b, W1, W2, k, cf, dy, 0.7, 0.3, round_fp32=False)
    monkeypatch.undo()                       # the finite differences use the true forward
    with pytest.raises(AssertionError):
        _fd_check(args, 0.7, 0.3, planted, n_coords=12, seed=7)
