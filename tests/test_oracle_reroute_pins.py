"""Pins of the oracle's rerouting of dropped assignments (CPU only).

`reroute` follows the reading of "dropped or routed to alternative experts"
([blog] "Expert Capacity") stated in its docstring.  It is pinned by
  - two hand-worked cases (tests/golden/reroute.json), exact integers;
  - brute force against an independent restatement over every small input: for
    each expert, the accepted second-chance offers are the first (C - kept rows)
    offers to it in (choice rank, token) order, where each token's alternatives
    come from a stable sort of its logits;
  - invariants: capacity holds, primary-kept choices are untouched, a token is
    never served twice by one expert, nothing changes when nothing was dropped
    or when no token has an unchosen expert (k = E), and rerouting keeps at
    least as many rows as dropping.
A planted-mistake test checks that each plausible wrong variant fails a pin.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle as O
import oracle.moe_oracle as M

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    with open(os.path.join(HERE, "golden", "reroute.json")) as f:
        return json.load(f)


def test_reroute_golden_cases():
    d = _golden()
    assert d["cite"] and d["reading"]
    for case in d["cases"]:
        logits = np.array(case["logits"], dtype=np.float32)
        S, E = logits.shape
        rt = O.route(logits, case["k"], case["cf"], rerouting=True)
        ex = case["expect"]
        assert rt.C == ex["C"], case["name"]
        assert rt.slot0.tolist() == ex["slot0"], case["name"]
        assert rt.dest.tolist() == ex["dest"], case["name"]
        assert rt.slot.tolist() == ex["slot"], case["name"]
        assert rt.n.tolist() == ex["n"], case["name"]


def _reroute_by_sorting(logits, ids, slot, cnt, C):
    """Independent restatement: alternatives from a stable descending sort of each
    token's logits; per expert, the first (C - kept) offers in (r, t) order win."""
    l = np.asarray(logits, dtype=np.float64)
    S, k = ids.shape
    E = l.shape[1]
    order = np.argsort(-l, axis=1, kind="stable")        # ties keep the lower index first
    offers = {e: [] for e in range(E)}
    for r in range(k):
        for t in range(S):
            if slot[t, r] >= 0:
                continue
            j = int(np.sum(slot[t, :r] < 0))
            if k + j < E:
                offers[int(order[t, k + j])].append((r, t))
    dest, out = ids.copy(), slot.copy()
    n = np.minimum(cnt, C).astype(np.int64)
    for e, lst in offers.items():
        room = max(0, C - int(n[e]))
        for i, (r, t) in enumerate(sorted(lst)[:room]):
            out[t, r] = n[e] + i
            dest[t, r] = e
        n[e] += min(room, len(lst))
    return dest, out, n


def _check_one(logits, k, cf):
    rt = O.route(logits, k, cf, rerouting=True)
    dest, slot, n = _reroute_by_sorting(logits, rt.ids, rt.slot0, rt.cnt, rt.C)
    assert np.array_equal(rt.dest, dest) and np.array_equal(rt.slot, slot) and np.array_equal(rt.n, n)
    return rt


def test_reroute_brute_force_small():
    count = 0
    for S, E, k in ((3, 3, 1), (3, 3, 2), (4, 4, 2), (3, 4, 3), (5, 3, 2)):
        base = np.arange(E, dtype=np.float32)
        perms = list(itertools.permutations(range(E)))
        rng = np.random.default_rng(S * 100 + E * 10 + k)
        for _ in range(120):
            rows = [perms[i] for i in rng.integers(0, len(perms), S)]
            logits = np.array([[base[p] for p in row] for row in rows], dtype=np.float32)
            if rng.random() < 0.3:                             # ties
                logits = np.floor(logits / 2)
            for C in range(0, S * k + 1):
                cf = C * E / (k * S) if C else 0.01
                rt = _check_one(logits, k, cf)
                count += 1
    assert count > 3000


def test_reroute_invariants_random():
    rng = np.random.default_rng(7)
    for _ in range(60):
        S, E = int(rng.integers(1, 60)), int(rng.integers(2, 12))
        k = int(rng.integers(1, E + 1))
        cf = float(rng.choice([0.25, 0.5, 0.8, 1.0, 1.5]))
        logits = (rng.standard_normal((S, E)) + 1.5 * np.log(1.0 / np.arange(1, E + 1))).astype(np.float32)
        rt = _check_one(logits, k, cf)
        C = rt.C
        kept0 = rt.slot0 >= 0
        # primary-kept choices keep their expert and slot
        assert np.array_equal(rt.slot[kept0], rt.slot0[kept0]) and np.array_equal(rt.dest[kept0], rt.ids[kept0])
        # capacity and dense slots per expert
        for e in range(E):
            s = np.sort(rt.slot[(rt.dest == e) & (rt.slot >= 0)])
            assert np.array_equal(s, np.arange(len(s))) and len(s) == rt.n[e] <= C
        # a token is served by distinct experts; a rerouted choice goes to an unchosen expert
        for t in range(S):
            served = rt.dest[t][rt.slot[t] >= 0]
            assert len(set(served.tolist())) == len(served)
            moved = (rt.dest[t] != rt.ids[t])
            assert not np.isin(rt.dest[t][moved], rt.ids[t]).any()
        assert (rt.slot >= 0).sum() >= kept0.sum()
        no = O.route(logits, k, cf)
        assert np.array_equal(no.slot, rt.slot0) and np.array_equal(no.ids, rt.ids)


def test_reroute_changes_nothing_without_drops_or_alternatives():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((40, 6)).astype(np.float32)
    rt = O.route(logits, 2, 6 / 2, rerouting=True)            # cf = E/k: nothing can drop
    assert np.array_equal(rt.dest, rt.ids) and np.array_equal(rt.slot, rt.slot0)
    rt = O.route(logits, 6, 0.3, rerouting=True)              # k = E: no unchosen expert
    assert (rt.slot0 < 0).any()
    assert np.array_equal(rt.dest, rt.ids) and np.array_equal(rt.slot, rt.slot0)


def test_rerouted_forward_uses_the_serving_expert():
    """y of a rerouted token is its gate weight times the serving expert's FFN."""
    d = _golden()["cases"][1]
    logits = np.array(d["logits"], dtype=np.float32)
    S, E = logits.shape
    rng = np.random.default_rng(0)
    M_, H = 4, 6
    x = rng.standard_normal((S, M_))
    W1 = rng.standard_normal((E, M_, H))
    W2 = rng.standard_normal((E, H, M_))
    rt = O.forward(x, None, None, W1, W2, d["k"], d["cf"], logits=logits, rerouting=True)
    # token 1: first choice dropped for good, second served by expert 4 with weight g_1
    g1 = 1.0 / (1.0 + np.exp(1.0))
    want = g1 * (np.maximum(x[1] @ W1[4], 0) @ W2[4])
    assert np.allclose(rt.y[1], want, rtol=1e-12, atol=1e-12)
    assert np.allclose(rt.gates[1], [1 - g1, g1], rtol=1e-12)


# ---- planted mistakes -------------------------------------------------------------

def _mut_same_alternative(logits, ids, slot, cnt, C):
    # every dropped choice of a token is offered the same (k-th ranked) expert
    l = np.asarray(logits)
    S, k = ids.shape
    ranking = O.top_k(l, l.shape[1])
    n = np.minimum(cnt, C).astype(np.int64)
    dest, out = ids.astype(np.int32).copy(), np.array(slot, dtype=np.int32, copy=True)
    for r in range(k):
        for t in range(S):
            if slot[t, r] >= 0 or k >= l.shape[1]:
                continue
            a = ranking[t, k]
            if n[a] < C:
                out[t, r], dest[t, r] = n[a], a
                n[a] += 1
    return dest, out, n


def _mut_token_major(logits, ids, slot, cnt, C):
    l = np.asarray(logits)
    S, k = ids.shape
    E = l.shape[1]
    ranking = O.top_k(l, E)
    n = np.minimum(cnt, C).astype(np.int64)
    dest, out = ids.astype(np.int32).copy(), np.array(slot, dtype=np.int32, copy=True)
    for t in range(S):
        j = 0
        for r in range(k):
            if slot[t, r] >= 0:
                continue
            if k + j < E:
                a = ranking[t, k + j]
                if n[a] < C:
                    out[t, r], dest[t, r] = n[a], a
                    n[a] += 1
            j += 1
    return dest, out, n


def _mut_ignores_primary_rows(logits, ids, slot, cnt, C):
    # free capacity counted from zero instead of from the rows the pass kept
    return M.__dict__["_orig_reroute"](logits, ids, slot, np.zeros_like(cnt), C)


PINS = [test_reroute_golden_cases, test_reroute_brute_force_small, test_reroute_invariants_random,
        test_reroute_changes_nothing_without_drops_or_alternatives, test_rerouted_forward_uses_the_serving_expert]


@pytest.mark.parametrize("mutant", [_mut_same_alternative, _mut_token_major, _mut_ignores_primary_rows],
                         ids=lambda m: m.__name__)
def test_pins_catch_planted_reroute_mistake(mutant, monkeypatch):
    monkeypatch.setitem(M.__dict__, "_orig_reroute", M.reroute)
    monkeypatch.setattr(M, "reroute", mutant)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutant.__name__}"
