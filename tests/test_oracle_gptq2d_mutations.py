"""Plant plausible mistakes in a copy of the GPTQ-2D oracle; a pin must fail.

Each mutant is oracle/gptq2d_oracle.py with one edit (a transposed factor, a
dropped scaling, feedback from the wrong rows, a lost accumulation, a skipped
entry), loaded as a separate module on the CPU.  The pins are the same kinds of
checks as in test_oracle_gptq2d.py: the hand-derived 2x2 examples, the identity
with the one-dimensional column loop on vec(W), and the closed forms.
"""
import inspect
import json
import os
import types
from fractions import Fraction

import numpy as np
import pytest

import oracle  # noqa: F401  (the mutants import the one-sided factor from it)
from oracle import gptq2d_oracle
from oracle import gptq_oracle as go

MUTATIONS = {
    "left factor transposed in the decision": (
        'np.einsum("ki,ki->i", UL[:, ii], M[:, jj])', 'np.einsum("ik,ki->i", UL[ii, :], M[:, jj])'),
    "right factor column instead of row": ("M[ii, :] += e[:, None] * UR[jj, :]", "M[ii, :] += e[:, None] * UR[:, jj].T"),
    "error not scaled by UR_jj": ("e = (wt - dq) / (UL[ii, ii] * UR[jj, jj])", "e = (wt - dq) / UL[ii, ii]"),
    "feedback from the own row only": (
        'np.einsum("ki,ki->i", UL[:, ii], M[:, jj])', "UL[ii, ii] * M[ii, jj]"),
    "errors not accumulated": ("M[ii, :] += e[:, None]", "M[ii, :] = e[:, None]"),
    "last row skipped": ("hi = min(d, m - 1)", "hi = min(d, m - 2)"),
    "sign of the feedback": ("wt = W[ii, jj] - np.einsum", "wt = W[ii, jj] + np.einsum"),
}


def _mutant(edit):
    src = inspect.getsource(gptq2d_oracle)
    old, new = edit
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.gptq2d_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "gptq2d_mutant", "exec"), mod.__dict__)
    return mod


def _fl(M):
    return np.array([[float(Fraction(x)) for x in r] for r in M])


def _pin_worked_examples(g2):
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "golden", "gptq2d_examples.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        res = g2.gptq2d_from_grams(_fl(case["W"]), _fl(case["HL"]), _fl(case["HR"]))
        assert np.array_equal(res["codes"], np.array(case["codes"]))
        assert np.allclose(res["decision"], _fl(case["decision_values"]), atol=1e-12)


def _spd(rng, n):
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    return (Q * np.geomspace(1.0, 20.0, n)) @ Q.T


def _pin_vec_identity(g2):
    rng = np.random.default_rng(11)
    m, n = 4, 5
    HL, HR = _spd(rng, m), _spd(rng, n)
    W = rng.uniform(-3, 3, (m, n))
    res = g2.gptq2d_from_grams(W, HL, HR, 0.7)
    codes, _, E = go.gptq_core(W.reshape(1, -1), go.inverse_factor(np.kron(HL, HR)), 1, go.IntegerGrid(0.7))
    assert np.array_equal(codes.reshape(m, n), res["codes"])
    assert np.allclose(E.reshape(m, n), res["E"], atol=1e-10)


def _pin_closed_forms(g2):
    rng = np.random.default_rng(12)
    m, n = 9, 6
    HL, HR = _spd(rng, m), _spd(rng, n)
    W = rng.standard_normal((m, n))
    res = g2.gptq2d_from_grams(W, HL, HR, 0.5)
    assert np.allclose(W - res["deq"], res["UL"].T @ res["E"] @ res["UR"], atol=1e-10)
    assert np.isclose(g2.two_sided_objective(W, res["deq"], HL, HR), np.sum(res["E"] ** 2), rtol=1e-9)


PINS = [_pin_worked_examples, _pin_vec_identity, _pin_closed_forms]


def test_pins_pass_on_the_oracle():
    for pin in PINS:
        pin(gptq2d_oracle)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_each_mutation_is_caught(name):
    g2 = _mutant(MUTATIONS[name])
    failures = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(g2)
        except Exception:  # an assertion, or the mutant crashing
            failures += 1
    assert failures > 0, f"no pin catches: {name}"
