"""Plant plausible mistakes in a copy of the oracle and check that a pin fails.

Each mutant is the oracle's source with one edit (a transposed operand, a flipped
sign, a dropped term, a wrong index or order), loaded as a separate module on
the CPU.  The pins re-run against the mutant are the same kinds of checks as in
test_oracle_pins.py: hand-derived worked examples, block-size invariance,
diagonal-H = round-to-nearest, Babai equivalence and the closed-form identities.
"""
import inspect
import json
import os
import types
from fractions import Fraction

import numpy as np
import pytest

from oracle import gptq_oracle
from tests.lattice_ref import babai_nearest_plane

MUTATIONS = {
    "transposed in-block row": ("U[col, col + 1:i2])", "U[col + 1:i2, col])"),
    "flipped in-block sign": ("Wb[:, j + 1:] -= np.outer", "Wb[:, j + 1:] += np.outer"),
    "dropped trailing update": ("        W[:, i2:] -= E[:, i1:i2] @ U[i1:i2, i2:]\n", "        pass\n"),
    "error not scaled by U_jj": ("e = (Wb[:, j] - dq) / U[col, col]", "e = (Wb[:, j] - dq)"),
    "trailing uses transposed U": ("        W[:, i2:] -= E[:, i1:i2] @ U[i1:i2, i2:]\n", "        W[:, i2:] -= E[:, i1:i2] @ U[i2:, i1:i2].T\n"),
    "group params from stale weights": ("cur = Wb[:, j:hi - i1]", "cur = W[:, col:hi]"),
    "zero point sign": ("zero = np.rint(-xmin / scale)", "zero = np.rint(xmin / scale)"),
    "grid not widened to 0": ("xmin = np.minimum(cols.min(axis=1), 0.0)", "xmin = cols.min(axis=1)"),
    "ascending act-order": ('perm = np.argsort(-key, kind="stable")', 'perm = np.argsort(key, kind="stable")'),
    "damping from max": ("lam = float(damp) * float(np.mean(np.diag(H)))", "lam = float(damp) * float(np.max(np.diag(H)))"),
    "lower factor instead of upper": ("return _cholesky(Hinv).T", "return _cholesky(Hinv)"),
    "reversed factor not reversed back": ("return _lower_inverse(Lr)[::-1, ::-1].copy()", "return _lower_inverse(Lr).T.copy()"),
    "matvec groups interleaved": ("else np.arange(n) // G", "else np.arange(n) % max(n // G, 1)"),
    "matvec zero point added": ("Q = s * (codes - z)", "Q = s * (codes + z)"),
    "matvec transposed product": ("return x @ Q.T", "return (Q @ x.T).T[:, ::-1]"),
}


def _mutant(edit):
    src = inspect.getsource(gptq_oracle)
    old, new = edit
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _golden(name):
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "golden", name)) as f:
        return json.load(f)


def _pin_worked_examples(go):
    for case in _golden("worked_examples.json")["cases"]:
        H = np.array([[float(Fraction(x)) for x in r] for r in case["H"]])
        w = np.array([float(Fraction(x)) for x in case["w"]])
        for key in ("forward", "backward"):
            perm = np.array(case[key]["order"])
            U = go.inverse_factor(H[np.ix_(perm, perm)])
            codes, _, _ = go.gptq_core(w[perm][None, :], U, 1, go.IntegerGrid(1.0))
            out = np.zeros(len(w))
            out[perm] = codes[0]
            assert out.tolist() == case[key]["codes"]


def _pin_grid(go):
    for case in _golden("grid_examples.json")["cases"]:
        maxq = (1 << case["bits"]) - 1
        w = np.array(case["w"])[None, :]
        s, z = go.group_params(w, maxq)
        q, _ = go.quantize_values(w[0], s[0], z[0], maxq)
        assert q.tolist() == case["codes"]


def _inputs(seed, n=64):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((300, n)) * np.exp(rng.standard_normal(n))[None, :]
    W = 0.02 * rng.standard_normal((12, n))
    return W, X


def _pin_block_invariance(go):
    W, X = _inputs(1)
    a = go.gptq_layer(W, X=X, bits=3, group=16, damp=0.01, block=16)
    b = go.gptq_layer(W, X=X, bits=3, group=16, damp=0.01, block=64)
    assert np.array_equal(a["codes"], b["codes"])


def _pin_identities(go):
    W, X = _inputs(2)
    out = go.gptq_layer(W, X=X, bits=3, group=16, damp=0.01, block=32, act_order=True)
    perm, U = out["perm"], out["U"]
    # the factor itself, both routes
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.allclose(go.inverse_factor_reversed(out["H"]), U, atol=1e-9)
    assert np.allclose(U.T @ U @ out["H"], np.eye(U.shape[0]), atol=1e-8)
    Qp = out["deq"][:, perm]
    assert np.allclose(out["W"] - Qp, out["E"] @ U, atol=1e-10)
    G = 16
    for g in range(W.shape[1] // G):
        c = g * G
        cur = out["W"][:, c:c + G] - out["E"][:, :c] @ U[:c, c:c + G]
        s, _ = gptq_oracle.group_params(cur, 7)
        assert np.allclose(out["scales"][:, g], s, rtol=1e-10)
    # act-order key is descending diag(H)
    H = gptq_oracle.hessian(X)
    assert np.array_equal(perm, np.argsort(-np.diag(H), kind="stable"))
    # damping closed form: H = I, damp 0.5 -> U = I / sqrt(1.5)
    prep = go.prepare(np.diag([1.0, 3.0]), np.zeros((1, 2)), 0.5, False)
    assert np.isclose(prep["lam"], 1.0)


def _pin_babai(go):
    rng = np.random.default_rng(5)
    n = 7
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    H = (Q * np.exp(rng.uniform(0, 3, n))) @ Q.T
    w = rng.standard_normal(n)
    perm = np.arange(n)[::-1]
    U = go.inverse_factor_reversed(H[np.ix_(perm, perm)])
    codes, _, _ = go.gptq_core(w[perm][None, :], U, 128, go.IntegerGrid(0.5))
    got = np.zeros(n)
    got[perm] = codes[0]
    B = np.linalg.cholesky(H).T
    c, _ = babai_nearest_plane(0.5 * B, B @ w)
    assert np.array_equal(got, c)
    # the scaled errors reproduce the lattice distance (loss identity)
    d = w - 0.5 * c
    _, _, E = go.gptq_core(w[perm][None, :], U, 128, go.IntegerGrid(0.5))
    assert np.isclose(np.sum(E ** 2), d @ H @ d, rtol=1e-9)


def _pin_diag_rtn(go):
    rng = np.random.default_rng(3)
    W = 0.02 * rng.standard_normal((8, 64))
    out = go.gptq_layer(W, H=np.diag(rng.uniform(0.5, 2, 64)), bits=4, group=16, damp=0.01, block=32)
    ref = gptq_oracle.rtn_quantize(W, 4, 16)
    assert np.array_equal(out["codes"], ref["codes"])


def _pin_matvec(go):
    for case in _golden("matvec_examples.json")["cases"]:
        packed = np.array([[int(w, 16) for w in row] for row in case["packed"]], dtype=np.uint32)
        y = go.dequant_matvec(packed, np.array(case["scales"]), np.array(case["zeros"]), case["n"], case["bits"],
                              case["group"], np.array(case["x"]), case.get("g_idx"))
        assert np.array_equal(y, np.array(case["y"]))


PINS = [_pin_worked_examples, _pin_grid, _pin_block_invariance, _pin_identities, _pin_babai, _pin_diag_rtn,
        _pin_matvec]


def test_pins_pass_on_the_oracle():
    for pin in PINS:
        pin(gptq_oracle)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_each_mutation_is_caught(name):
    go = _mutant(MUTATIONS[name])
    failures = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(go)
        except Exception:  # an assertion, or the mutant crashing
            failures += 1
    assert failures > 0, f"no pin catches: {name}"
