"""Planted mistakes in the oracle must each be caught by some pin (CPU only).

Every mutant below replaces one oracle function with a plausible wrong version
(a flipped tie rule, a dropped normalisation, a token-major scan, ...).  The pin
tests are then run against the mutated oracle and at least one of them must
fail.  Nothing here touches the CUDA path.
"""
import math

import numpy as np
import pytest

import oracle.moe_oracle as M
import tests.test_oracle_pins as P

PINS = [getattr(P, n) for n in dir(P) if n.startswith("test_")]


def _mut_topk_high_ties(logits, k):
    l = np.array(logits, dtype=np.float32)[:, ::-1].copy()
    E = l.shape[1]
    ids = np.zeros((l.shape[0], k), np.int32)
    for r in range(k):
        j = np.argmax(l, axis=1)
        ids[:, r] = E - 1 - j
        l[np.arange(l.shape[0]), j] = -np.inf
    return ids


def _mut_gates_unnormalised(p, ids):
    return np.take_along_axis(M._f64(p), ids.astype(np.int64), axis=1)


def _mut_slots_token_major(ids, E, C):
    S, k = ids.shape
    slot = np.full((S, k), -1, np.int32)
    cnt = np.zeros(E, np.int64)
    for t in range(S):
        for r in range(k):
            e = ids[t, r]
            if cnt[e] < C:
                slot[t, r] = cnt[e]
            cnt[e] += 1
    return slot, cnt


def _mut_slots_second_choice_uses_raw_count(ids, E, C):
    # drops are not counted towards later positions (off by the dropped ones)
    S, k = ids.shape
    slot = np.full((S, k), -1, np.int32)
    cnt = np.zeros(E, np.int64)
    for r in range(k):
        for t in range(S):
            e = ids[t, r]
            if cnt[e] < C:
                slot[t, r] = cnt[e]
                cnt[e] += 1
    return slot, cnt


def _mut_capacity_floor_plus_one(S, E, k, cf):
    return int(math.floor(cf * k * S / E)) + 1


def _mut_capacity_round(S, E, k, cf):
    return int(round(cf * k * S / E))


def _mut_aux_all_choices(p, ids, lse, E):
    p = M._f64(p)
    S = p.shape[0]
    if S == 0:
        return 0.0, 0.0, np.zeros(E), np.zeros(E)
    P = p.mean(0)
    f = np.bincount(np.asarray(ids).ravel(), minlength=E) / (S * ids.shape[1])
    return float(E * np.sum(f * P)), float(np.mean(M._f64(lse) ** 2)), f, P


def _mut_aux_z_not_squared(p, ids, lse, E):
    a, _, f, P = M.__dict__["_orig_aux"](p, ids, lse, E)
    return a, float(np.mean(M._f64(lse))) if len(lse) else 0.0, f, P


def _mut_aux_no_E(p, ids, lse, E):
    a, z, f, P = M.__dict__["_orig_aux"](p, ids, lse, E)
    return a / E, z, f, P


def _mut_combine_renormalise(ybuf, ids, gates, slot):
    g = np.where(slot >= 0, gates, 0.0)
    s = g.sum(1, keepdims=True)
    g = np.where(s > 0, g / np.where(s > 0, s, 1), 0)
    return M.__dict__["_orig_combine"](ybuf, ids, g, slot)


def _mut_ffn_relu_on_output(rows, W1e, W2e):
    return np.maximum((M._f64(rows) @ M._f64(W1e)) @ M._f64(W2e), 0.0)


def _mut_ffn_no_relu(rows, W1e, W2e):
    return (M._f64(rows) @ M._f64(W1e)) @ M._f64(W2e)


def _mut_softmax_wrong_sign(logits):
    p, lse = M.__dict__["_orig_softmax"](-M._f64(logits))
    return p, lse


def _mut_logits_transposed_bias(x, Wg, bias=None):
    l = (M._f64(x) @ M._f64(Wg)).astype(np.float32)
    if bias is not None:
        l = l - np.asarray(M._f64(bias), np.float32)
    return l


def _mut_logits_fp16(x, Wg, bias=None):
    l = (M._f64(x) @ M._f64(Wg)).astype(np.float16).astype(np.float32)
    if bias is not None:
        l = l + np.asarray(M._f64(bias), np.float32)
    return l


def _mut_dispatch_wrong_rank(x, ids, slot, E, C):
    return M.__dict__["_orig_dispatch"](x, ids[:, ::-1].copy(), slot, E, C)


MUTANTS = {
    "top_k": [_mut_topk_high_ties],
    "normalized_gates": [_mut_gates_unnormalised],
    "assign_slots": [_mut_slots_token_major, _mut_slots_second_choice_uses_raw_count],
    "capacity": [_mut_capacity_floor_plus_one, _mut_capacity_round],
    "aux_losses": [_mut_aux_all_choices, _mut_aux_z_not_squared, _mut_aux_no_E],
    "combine": [_mut_combine_renormalise],
    "expert_ffn": [_mut_ffn_relu_on_output, _mut_ffn_no_relu],
    "softmax_stats": [_mut_softmax_wrong_sign],
    "gate_logits": [_mut_logits_transposed_bias, _mut_logits_fp16],
    "dispatch": [_mut_dispatch_wrong_rank],
}

CASES = [(fn, m) for fn, ms in MUTANTS.items() for m in ms]


@pytest.mark.parametrize("fn,mutant", CASES, ids=[m.__name__ for _, m in CASES])
def test_pins_catch_planted_mistake(fn, mutant, monkeypatch):
    monkeypatch.setitem(M.__dict__, "_orig_aux", M.aux_losses)
    monkeypatch.setitem(M.__dict__, "_orig_combine", M.combine)
    monkeypatch.setitem(M.__dict__, "_orig_softmax", M.softmax_stats)
    monkeypatch.setitem(M.__dict__, "_orig_dispatch", M.dispatch)
    monkeypatch.setattr(M, fn, mutant)
    monkeypatch.setattr(P.O, fn, mutant, raising=False)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mutant.__name__} in {fn}"
