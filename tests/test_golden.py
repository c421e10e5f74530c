"""The oracle against the hand-worked examples in tests/golden/ (CPU only).

The source pages print no worked example.  Each fixture works a small case out by
hand from the definitions (its `cite` and `reading` fields name the passage and
the reading used) and states the expected values exactly: integers, fractions, or
closed forms in exp and log.  Nothing in a fixture comes from the oracle or the
CUDA path, so a wrong index, sign, normalisation or slot order in the oracle
fails here.
"""
import json
import math
import pathlib
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = pathlib.Path(__file__).parent / "golden"


def value(expr) -> float:
    """A fixture number: an int, a float, or a string in +-*/, **, exp and log."""
    if isinstance(expr, (int, float)):
        return float(expr)
    if "/" in expr and not any(c.isalpha() for c in expr):
        return float(Fraction(expr))
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp, "log": math.log}))


def values(a) -> np.ndarray:
    return np.array([[value(v) for v in row] for row in a]) if isinstance(a[0], list) else \
        np.array([value(v) for v in a])


def load(name):
    with open(GOLDEN / name) as fh:
        return json.load(fh)


def check_route(rt, exp, E):
    assert rt.C == exp["C"]
    assert np.array_equal(rt.ids, np.array(exp["ids"]))
    assert np.array_equal(rt.slot, np.array(exp["slot"]))
    assert np.array_equal(rt.cnt, np.array(exp["cnt"]))
    if "n" in exp:
        assert np.array_equal(rt.n, np.array(exp["n"]))
    np.testing.assert_allclose(rt.gates, values(exp["gates"]), rtol=1e-12, atol=1e-15)
    if "f" in exp:
        np.testing.assert_allclose(rt.f, values(exp["f"]), rtol=1e-12, atol=1e-15)
    if "P" in exp:
        np.testing.assert_allclose(rt.P, values(exp["P"]), rtol=1e-12)
    if "l_aux" in exp:
        assert math.isclose(rt.l_aux, value(exp["l_aux"]), rel_tol=1e-12)
    if "z" in exp:
        assert math.isclose(rt.z, value(exp["z"]), rel_tol=1e-12)


def test_route_rank_major_fixture():
    g = load("route_rank_major.json")
    assert g["cite"] and g["reading"]
    logits = np.array(g["logits"], dtype=np.float64)
    rt = O.route(logits, g["k"], g["cf"])
    check_route(rt, g["expect"], g["E"])


@pytest.mark.parametrize("i", range(3))
def test_losses_and_gates_fixture(i):
    g = load("losses_and_gates.json")
    assert g["cite"] and g["reading"]
    case = g["cases"][i]
    logits = values(g["logits"])
    rt = O.route(logits, case["k"], case["cf"])
    check_route(rt, case["expect"], g["E"])


def test_backward_closed_form_fixture():
    g = load("backward_closed_form.json")
    assert g["cite"] and g["reading"]
    a = g["aux_and_z"]
    p, f, lse = values(a["p"]), values(a["f"]), values(a["lse"])
    np.testing.assert_allclose(O.aux_loss_backward(p, f, a["E"], a["S"]), values(a["expect_aux"]),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(O.z_loss_backward(p, lse, a["S"]), values(a["expect_z"]), rtol=1e-12)
    gt = g["gates"]
    dl = O.gates_backward(values(gt["gates"]), np.array(gt["ids"]), values(gt["dgate"]), gt["E"])
    np.testing.assert_allclose(dl, values(gt["expect"]), rtol=1e-12, atol=1e-15)
    fx = g["expert_ffn"]
    rows, W1, W2, dY = (values(fx[n]) for n in ("rows", "W1", "W2", "dY"))
    drows, dW1, dW2 = O.expert_ffn_backward(rows, rows @ W1, dY, W1, W2)
    np.testing.assert_allclose(drows, values(fx["expect_drows"]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dW1, values(fx["expect_dW1"]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dW2, values(fx["expect_dW2"]), rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- the fixtures catch plants
# The planted mistakes of the other pin files, restricted to those a routing, loss or
# step-gradient fixture can see (the fixtures have no ties, compute no logits and run no
# forward FFN, dispatch or combine): each must make at least one fixture test fail.
def _golden_pins():
    return [test_route_rank_major_fixture] + \
        [lambda i=i: test_losses_and_gates_fixture(i) for i in range(3)] + \
        [test_backward_closed_form_fixture]


def _planted():
    import tests.test_oracle_backward_pins as B
    import tests.test_oracle_mutations as MU
    fwd = [("normalized_gates", MU._mut_gates_unnormalised),
           ("assign_slots", MU._mut_slots_token_major),
           ("assign_slots", MU._mut_slots_second_choice_uses_raw_count),
           ("capacity", MU._mut_capacity_floor_plus_one),
           ("aux_losses", MU._mut_aux_all_choices),
           ("aux_losses", MU._mut_aux_z_not_squared),
           ("aux_losses", MU._mut_aux_no_E),
           ("softmax_stats", MU._mut_softmax_wrong_sign)]
    bwd = [(n, f) for n, fs in B.PLANTS.items() for f in fs]
    return fwd + bwd


PLANTED = _planted()


@pytest.mark.parametrize("fn,mutant", PLANTED, ids=[m.__name__ for _, m in PLANTED])
def test_fixtures_catch_planted_mistake(fn, mutant, monkeypatch):
    import oracle.moe_oracle as M
    monkeypatch.setitem(M.__dict__, "_orig_aux", M.aux_losses)
    monkeypatch.setitem(M.__dict__, "_orig_softmax", M.softmax_stats)
    monkeypatch.setattr(M, fn, mutant)
    monkeypatch.setattr(O, fn, mutant, raising=False)
    failed = []
    for pin in _golden_pins():
        try:
            pin()
        except Exception:
            failed.append(pin)
    assert failed, f"no fixture caught the planted mistake {mutant.__name__} in {fn}"
