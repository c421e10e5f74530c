"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test fixes one part of the oracle against something it does not compute
itself: a hand-worked example, a closed form of the definition, a library
routine (scipy) on a case that reduces to it, brute-force enumeration on tiny
inputs, or an invariant.  The expected values are written out by hand below;
none comes from the CUDA path.
"""
import itertools
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle as O

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- capacity
def test_capacity_hand_values():
    # the tiny workload states C = 80 for S=256, E=8, k=2, cf=1.25
    assert O.capacity(256, 8, 2, 1.25) == 80
    assert O.capacity(8192, 32, 2, 2.0) == 1024
    assert O.capacity(16384, 128, 2, 1.25) == 320
    assert O.capacity(65536, 64, 2, 1.0) == 2048
    assert O.capacity(16384, 256, 8, 1.25) == 640
    # ceil, not floor + 1 and not round
    assert O.capacity(10, 3, 2, 1.0) == 7      # 20/3 = 6.67
    assert O.capacity(12, 4, 2, 1.0) == 6      # exactly 6
    assert O.capacity(1, 8, 2, 0.1) == 1       # 0.025 -> 1
    assert O.capacity(100, 4, 1, 0.5) == 13    # 12.5


# ---------------------------------------------------------------- logits
def test_logits_hand_example():
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    Wg = np.array([[1.0, 0.0, 1.0], [0.0, 1.0, 1.0]])
    assert O.gate_logits(x, Wg).tolist() == [[1, 2, 3], [3, 4, 7]]
    b = np.array([0.5, -1.0, 0.0])
    assert O.gate_logits(x, Wg, b).tolist() == [[1.5, 1, 3], [3.5, 3, 7]]
    assert O.gate_logits(x, Wg).dtype == np.float32


def test_logits_one_hot_columns_copy_x():
    x = RNG.standard_normal((7, 5)).astype(np.float32)
    Wg = np.zeros((5, 3), dtype=np.float32)
    Wg[4, 0] = Wg[0, 1] = Wg[2, 2] = 1.0
    l = O.gate_logits(x, Wg)
    assert np.array_equal(l, x[:, [4, 0, 2]])


def test_logits_rounded_once_to_fp32():
    # 1 + 2^-30 is not representable in fp32; the float64 product is rounded once
    x = np.array([[1.0, 2.0 ** -30]])
    Wg = np.array([[1.0], [1.0]])
    assert O.gate_logits(x, Wg)[0, 0] == np.float32(1.0)
    x = np.array([[1.0, 2.0 ** -23]])
    assert O.gate_logits(x, Wg)[0, 0] == np.float32(1.0 + 2.0 ** -23)


# ---------------------------------------------------------------- softmax
def test_softmax_closed_forms():
    l = np.full((3, 5), 2.5, dtype=np.float32)
    p, lse = O.softmax_stats(l)
    assert np.allclose(p, 0.2, rtol=0, atol=1e-15)
    assert np.allclose(lse, 2.5 + math.log(5), rtol=0, atol=1e-14)
    d = 1.75
    p, lse = O.softmax_stats(np.array([[d, 0.0]], dtype=np.float32))
    assert abs(p[0, 0] - 1.0 / (1.0 + math.exp(-d))) < 1e-15
    assert abs(lse[0] - math.log(1.0 + math.exp(d))) < 1e-14


def test_softmax_matches_scipy():
    l = (RNG.standard_normal((50, 17)) * 4).astype(np.float32)
    p, lse = O.softmax_stats(l)
    assert np.allclose(p, softmax(l.astype(np.float64), axis=1), rtol=1e-13, atol=0)
    assert np.allclose(lse, logsumexp(l.astype(np.float64), axis=1), rtol=1e-14, atol=0)


# ---------------------------------------------------------------- top-k
def test_topk_all_permutations():
    for E in (3, 4):
        for perm in itertools.permutations(range(E)):
            l = np.array([perm], dtype=np.float32)
            for k in range(1, E + 1):
                ids = O.top_k(l, k)[0].tolist()
                want = [perm.index(E - 1 - r) for r in range(k)]
                assert ids == want, (perm, k)


def test_topk_ties_to_lower_index():
    assert O.top_k(np.zeros((1, 6), np.float32), 3)[0].tolist() == [0, 1, 2]
    assert O.top_k(np.array([[1, 0, 1, 0]], np.float32), 2)[0].tolist() == [0, 2]
    assert O.top_k(np.array([[0, 1, 1, 1]], np.float32), 2)[0].tolist() == [1, 2]
    assert O.top_k(np.array([[-0.0, 0.0]], np.float32), 1)[0].tolist() == [0]
    assert O.top_k(np.array([[0.0, -0.0]], np.float32), 2)[0].tolist() == [0, 1]


def test_topk_property_on_tie_heavy_rows():
    l = RNG.integers(0, 3, size=(400, 7)).astype(np.float32)
    for k in (1, 2, 3, 7):
        ids = O.top_k(l, k)
        for t in range(l.shape[0]):
            sel = ids[t].tolist()
            assert len(set(sel)) == k
            rest = [j for j in range(7) if j not in sel]
            for j in sel:
                for jj in rest:
                    assert l[t, j] > l[t, jj] or (l[t, j] == l[t, jj] and j < jj)
            for a, b in zip(sel, sel[1:]):
                assert l[t, a] > l[t, b] or (l[t, a] == l[t, b] and a < b)


# ---------------------------------------------------------------- gates
def test_gates_two_way_closed_form():
    l = (RNG.standard_normal((40, 6)) * 2).astype(np.float32)
    p, _ = O.softmax_stats(l)
    ids = O.top_k(l, 2)
    g = O.normalized_gates(p, ids)
    l0 = l[np.arange(40), ids[:, 0]].astype(np.float64)
    l1 = l[np.arange(40), ids[:, 1]].astype(np.float64)
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-13, atol=0)
    assert np.allclose(g.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(g[:, 0] >= g[:, 1])
    # equal to a softmax over the selected logits (library routine)
    for k in (1, 3, 6):
        ids = O.top_k(l, k)
        g = O.normalized_gates(p, ids)
        sel = np.take_along_axis(l.astype(np.float64), ids.astype(np.int64), 1)
        assert np.allclose(g, softmax(sel, axis=1), rtol=1e-12, atol=0)


def test_gates_hand_example():
    # p proportional to [1, 2, 4]: top-2 is [2, 1], gates 4/6 and 2/6
    l = np.array([[0.0, math.log(2.0), math.log(4.0)]], dtype=np.float32)
    rt = O.route(l, 2, 10.0)
    assert rt.ids[0].tolist() == [2, 1]
    assert np.allclose(rt.gates[0], [2 / 3, 1 / 3], rtol=1e-6)


# ---------------------------------------------------------------- slots
def _slots_by_sorting(ids, E, C):
    """Independent restatement: sort each expert's (rank, token) pairs; the first C are kept."""
    S, k = ids.shape
    slot = -np.ones((S, k), dtype=np.int64)
    cnt = np.zeros(E, dtype=np.int64)
    for e in range(E):
        pairs = sorted((r, t) for t in range(S) for r in range(k) if ids[t, r] == e)
        cnt[e] = len(pairs)
        for pos, (r, t) in enumerate(pairs[:C]):
            slot[t, r] = pos
    return slot, cnt


def test_slots_brute_force():
    cases = 0
    for E, k, S in ((3, 1, 4), (3, 2, 4), (2, 2, 3), (4, 2, 3), (2, 1, 5)):
        choices = list(itertools.permutations(range(E), k))
        for combo in itertools.product(choices, repeat=S):
            ids = np.array(combo, dtype=np.int32).reshape(S, k)
            for C in range(1, S * k + 1):
                slot, cnt = O.assign_slots(ids, E, C)
                ws, wc = _slots_by_sorting(ids, E, C)
                assert np.array_equal(slot, ws) and np.array_equal(cnt, wc), (ids, C)
                cases += 1
    assert cases > 5000


def test_slots_invariants_random():
    for trial in range(20):
        S, E = 300, int(RNG.integers(2, 20))
        k = int(RNG.integers(1, min(E, 4) + 1))
        l = RNG.standard_normal((S, E)).astype(np.float32) + np.linspace(0, 3, E).astype(np.float32)
        ids = O.top_k(l, k)
        prev_kept = None
        for cf in (0.25, 0.5, 1.0, 1.5, float(E) / k):
            C = O.capacity(S, E, k, cf)
            slot, cnt = O.assign_slots(ids, E, C)
            n = np.minimum(cnt, C)
            assert cnt.sum() == S * k
            assert (slot >= 0).sum() == n.sum()
            for e in range(E):
                got = np.sort(slot[(ids == e) & (slot >= 0)])
                assert np.array_equal(got, np.arange(n[e]))       # slots 0..n_e-1, no repeats
            kept = slot >= 0
            if prev_kept is not None:
                assert np.all(kept[prev_kept])                      # monotone in cf
            prev_kept = kept
        assert np.all(kept)                                         # cf >= E/k keeps all


def test_slots_rank_major_hand_example():
    # two tokens, both choose [0, 1]; C = 1: t0 keeps both, t1 loses both
    ids = np.array([[0, 1], [0, 1]], dtype=np.int32)
    slot, cnt = O.assign_slots(ids, 2, 1)
    assert slot.tolist() == [[0, 0], [-1, -1]] and cnt.tolist() == [2, 2]
    # first choices of later tokens beat second choices of earlier tokens
    ids = np.array([[0, 1], [1, 0]], dtype=np.int32)
    slot, _ = O.assign_slots(ids, 2, 1)
    assert slot.tolist() == [[0, -1], [0, -1]]


# ---------------------------------------------------------------- expert FFN / dense layer
def _dense_ffn_loops(x, W1, W2):
    S, M = len(x), len(x[0])
    H = len(W1[0])
    y = [[0.0] * M for _ in range(S)]
    for t in range(S):
        h = [max(0.0, sum(x[t][i] * W1[i][j] for i in range(M))) for j in range(H)]
        for m in range(M):
            y[t][m] = sum(h[j] * W2[j][m] for j in range(H))
    return np.array(y)


def test_single_expert_layer_is_dense_ffn():
    S, M, H = 4, 3, 5
    x = RNG.standard_normal((S, M))
    Wg = RNG.standard_normal((M, 1))
    W1 = RNG.standard_normal((1, M, H))
    W2 = RNG.standard_normal((1, H, M))
    rt = O.forward(x, Wg, None, W1, W2, k=1, cf=1.0)
    assert rt.C == S and np.all(rt.slot[:, 0] == np.arange(S))
    assert np.allclose(rt.gates, 1.0)
    want = _dense_ffn_loops(x.tolist(), W1[0].tolist(), W2[0].tolist())
    assert np.allclose(rt.y, want, rtol=1e-13, atol=1e-13)
    l = rt.logits.astype(np.float64)[:, 0]
    assert abs(rt.l_aux - 1.0) < 1e-15
    assert abs(rt.z - np.mean(l ** 2)) < 1e-12


# ---------------------------------------------------------------- losses
def test_losses_hand_examples():
    # both tokens: p = [3/4, 1/4], top-1 = expert 0 -> f = [1, 0], P = [3/4, 1/4]
    l = np.array([[math.log(3.0), 0.0]] * 2, dtype=np.float32)
    rt = O.route(l, 1, 1.0)
    assert abs(rt.l_aux - 1.5) < 1e-7
    assert abs(rt.z - math.log(4.0) ** 2) < 1e-6
    # t0: p = [1/4, 3/4] -> top-1 expert 1; t1: tie -> expert 0
    l = np.array([[0.0, math.log(3.0)], [0.0, 0.0]], dtype=np.float32)
    rt = O.route(l, 1, 1.0)
    assert rt.ids[:, 0].tolist() == [1, 0]
    assert np.allclose(rt.P, [3 / 8, 5 / 8], rtol=1e-7)
    assert abs(rt.l_aux - 1.0) < 1e-7
    assert abs(rt.z - 2.5 * math.log(2.0) ** 2) < 1e-6
    assert O.route(np.zeros((0, 4), np.float32), 2, 1.0).l_aux == 0.0


def test_losses_extreme_one_hot():
    E = 4
    l = np.zeros((10, E), dtype=np.float32)
    l[:, 0] = 60.0
    rt = O.route(l, 2, 1.0)
    assert abs(rt.l_aux - E) < 1e-12 * E
    assert np.allclose(rt.lse, 60.0, rtol=1e-12)


# ---------------------------------------------------------------- whole layer closed forms
def _ffn(x, W1e, W2e):
    return np.maximum(x @ W1e, 0) @ W2e


def test_uniform_gating_closed_form():
    S, M, H, E, k, cf = 40, 6, 10, 5, 2, 1.0
    x = RNG.standard_normal((S, M))
    W1 = RNG.standard_normal((E, M, H))
    W2 = RNG.standard_normal((E, H, M))
    rt = O.forward(x, np.zeros((M, E)), None, W1, W2, k, cf)
    C = O.capacity(S, E, k, cf)            # 16
    assert C == 16
    assert np.all(rt.ids == np.arange(k))
    assert np.allclose(rt.gates, 1.0 / k, rtol=0, atol=1e-15)
    assert abs(rt.l_aux - 1.0) < 1e-15
    assert abs(rt.z - math.log(E) ** 2) < 1e-12
    want = np.zeros((S, M))
    want[:C] = sum(_ffn(x[:C], W1[r], W2[r]) for r in range(k)) / k
    assert np.allclose(rt.y, want, rtol=1e-12, atol=1e-12)


def test_partial_drop_is_not_renormalised():
    # E=2, k=2, S=3, cf=0.5 -> C=2.  t0, t1 prefer expert 0, t2 prefers expert 1.
    l3 = math.log(3.0)
    l = np.array([[l3, 0.0], [l3, 0.0], [0.0, l3]], dtype=np.float32)
    rt = O.route(l, 2, 0.5)
    assert rt.C == 2
    assert rt.slot.tolist() == [[0, 1], [1, -1], [0, -1]]
    ybuf = np.zeros((2, 2, 1))
    ybuf[0, :, 0] = [10.0, 20.0]
    ybuf[1, :, 0] = [100.0, 200.0]
    y = O.combine(ybuf, rt.ids, rt.gates, rt.slot)
    assert np.allclose(y[:, 0], [0.75 * 10 + 0.25 * 200, 0.75 * 20, 0.75 * 100], rtol=1e-6)


def test_dispatch_places_rows():
    ids = np.array([[1, 0], [1, 2], [0, 1]], dtype=np.int32)
    slot, _ = O.assign_slots(ids, 3, 2)
    x = np.arange(6, dtype=np.float64).reshape(3, 2)
    xbuf = O.dispatch(x, ids, slot, 3, 2)
    # expert 1: t0 (r=0) slot 0, t1 (r=0) slot 1, t2 (r=1) dropped
    assert xbuf[1].tolist() == [[0, 1], [2, 3]]
    assert xbuf[0].tolist() == [[4, 5], [0, 1]]      # t2 r=0 then t0 r=1
    assert xbuf[2].tolist() == [[2, 3], [0, 0]]


def test_permutation_equivariance_unbounded_capacity():
    S, M, H, E, k = 64, 8, 12, 6, 2
    x = RNG.standard_normal((S, M))
    Wg = RNG.standard_normal((M, E))
    W1 = RNG.standard_normal((E, M, H))
    W2 = RNG.standard_normal((E, H, M))
    pi = RNG.permutation(S)
    a = O.forward(x, Wg, None, W1, W2, k, E / k)
    b = O.forward(x[pi], Wg, None, W1, W2, k, E / k)
    assert np.allclose(b.y, a.y[pi], rtol=1e-12, atol=1e-12)
    # losses are permutation invariant at any capacity
    c = O.forward(x, Wg, None, W1, W2, k, 0.5)
    d = O.forward(x[pi], Wg, None, W1, W2, k, 0.5)
    assert abs(c.l_aux - d.l_aux) < 1e-12 and abs(c.z - d.z) < 1e-12


def test_positive_homogeneity():
    S, M, H, E, k = 50, 8, 12, 4, 2
    x = RNG.standard_normal((S, M))
    Wg = RNG.standard_normal((M, E))
    W1 = RNG.standard_normal((E, M, H))
    W2 = RNG.standard_normal((E, H, M))
    a = O.forward(x, Wg, None, W1, W2, k, 1.0)
    b = O.forward(x, Wg, None, 2.5 * W1, W2, k, 1.0)
    c = O.forward(x, Wg, None, W1, 0.5 * W2, k, 1.0)
    assert np.array_equal(a.slot, b.slot)
    assert np.allclose(b.y, 2.5 * a.y, rtol=1e-12, atol=1e-12)
    assert np.allclose(c.y, 0.5 * a.y, rtol=1e-12, atol=1e-12)


def test_sampled_outputs_match_full_forward():
    S, M, H, E, k = 90, 8, 12, 5, 2
    x = RNG.standard_normal((S, M))
    Wg = RNG.standard_normal((M, E))
    W1 = RNG.standard_normal((E, M, H))
    W2 = RNG.standard_normal((E, H, M))
    rt = O.forward(x, Wg, None, W1, W2, k, 0.8)
    assert (rt.slot < 0).any()
    tok = np.array([0, 5, 17, 33, 89])
    y = O.outputs_for_tokens(tok, x[tok], rt.ids, rt.gates, rt.slot, lambda e: (W1[e], W2[e]))
    assert np.allclose(y, rt.y[tok], rtol=1e-12, atol=1e-12)
