"""Pins for the GPTQ-2D oracle (two-sided rounding, anti-diagonal order).

Everything here comes from outside oracle/gptq2d_oracle.py:

* hand-derived 2x2 examples (tests/golden/gptq2d_examples.json), exact fractions;
* the statement of the GPTQ-2D abstract ("Daily Papers" page) that the
  one-dimensional algorithm run on vec(W) with the Kronecker Gram gives the
  identical rounded matrix: checked against the one-sided column loop (itself
  pinned by its own tests) in row-major and in column-major order, and against
  an exact sequential-conditional-minimisation run that never forms a factor;
* Babai's nearest plane on the Kronecker lattice (tests/lattice_ref.py, written
  independently; GPTQ = Babai abstract on the same page) and its error bound;
* brute-force closest vectors on tiny matrices;
* closed forms: W - Q = UL^T E UR and tr(HL D HR D^T) = sum e^2;
* special cases: an identity Gram on one side leaves the familiar one-sided
  problem on the other; two diagonal Grams give round-to-nearest.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import gptq2d_oracle as g2
from oracle import gptq_oracle as go
from tests.lattice_ref import babai_nearest_plane


def _random_spd(rng, n, cond=20.0):
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    ev = np.geomspace(1.0, cond, n)
    return (Q * ev) @ Q.T


def _frac(M):
    return [[Fraction(x) for x in r] for r in M]


def _fl(M):
    return np.array([[float(x) for x in r] for r in M])


def _solve_exact(A, b):
    """Gauss-Jordan elimination in exact fractions (A square, nonsingular)."""
    n = len(A)
    M = [list(A[i]) + [b[i]] for i in range(n)]
    for c in range(n):
        p = next(r for r in range(c, n) if M[r][c] != 0)
        M[c], M[p] = M[p], M[c]
        piv = M[c][c]
        M[c] = [x / piv for x in M[c]]
        for r in range(n):
            if r != c and M[r][c] != 0:
                f = M[r][c]
                M[r] = [x - f * y for x, y in zip(M[r], M[c])]
    return [M[i][n] for i in range(n)]


def _round_half_even(x):
    fl = x.numerator // x.denominator
    rem = x - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        return fl + 1
    return fl


def _sequential_exact(G, w):
    """Round w to integers coordinate by coordinate in index order; after each
    decision the free coordinates move to the minimiser of the quadratic with
    the decided ones held fixed (shift H_FF^-1 H_Fk d_k).  Exact fractions,
    no factorisation."""
    n = len(w)
    w = list(w)
    codes, decision = [], []
    for k in range(n):
        decision.append(w[k])
        q = _round_half_even(w[k])
        codes.append(q)
        d = w[k] - q
        F = list(range(k + 1, n))
        if F:
            shift = _solve_exact([[G[a][b] for b in F] for a in F], [G[a][k] for a in F])
            for idx, a in enumerate(F):
                w[a] += shift[idx] * d
    return codes, decision


def _kron_frac(A, B):
    return [[A[i][k] * B[j][l] for k in range(len(A)) for l in range(len(B))]
            for i in range(len(A)) for j in range(len(B))]


def _exact_objective(W, Q, HL, HR):
    m, n = len(W), len(W[0])
    D = [[W[i][j] - Q[i][j] for j in range(n)] for i in range(m)]
    return sum(HL[a][b] * D[b][j] * HR[j][k] * D[a][k]
               for a in range(m) for b in range(m) for j in range(n) for k in range(n))


# ---------------------------------------------------------------------------
# worked examples
# ---------------------------------------------------------------------------

def _cases(golden_dir):
    with open(os.path.join(golden_dir, "gptq2d_examples.json")) as f:
        return json.load(f)["cases"]


def test_worked_examples(golden_dir):
    for case in _cases(golden_dir):
        HL, HR, W = _frac(case["HL"]), _frac(case["HR"]), _frac(case["W"])
        # exact-arithmetic statements of the golden values
        assert _exact_objective(W, case["codes"], HL, HR) == Fraction(case["loss"]), case["name"]
        assert _exact_objective(W, case["rtn_codes"], HL, HR) == Fraction(case["rtn_loss"]), case["name"]
        codes, decision = _sequential_exact(_kron_frac(HL, HR), [x for r in W for x in r])
        assert codes == [c for r in case["codes"] for c in r], case["name"]
        assert decision == [Fraction(x) for r in case["decision_values"] for x in r], case["name"]
        # the oracle
        res = g2.gptq2d_from_grams(_fl(W), _fl(HL), _fl(HR))
        assert np.array_equal(res["codes"], np.array(case["codes"])), case["name"]
        assert np.allclose(res["decision"], _fl(_frac(case["decision_values"])), atol=1e-12)
        assert np.isclose(np.sum(res["E"] ** 2), float(Fraction(case["loss"])), rtol=1e-12)
        assert np.array_equal(np.rint(_fl(W)), np.array(case["rtn_codes"]))


# ---------------------------------------------------------------------------
# identity with the one-dimensional algorithm on vec(W)
# ---------------------------------------------------------------------------

def _problem(seed, max_dim=5):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(1, max_dim + 1))
    n = int(rng.integers(1, max_dim + 1))
    HL = _random_spd(rng, m)
    HR = _random_spd(rng, n)
    W = rng.uniform(-3, 3, (m, n))
    scale = float(rng.uniform(0.3, 1.2))
    return rng, m, n, HL, HR, W, scale


class _ClampedGrid(go.IntegerGrid):
    def __init__(self, scale, lo, hi):
        super().__init__(scale)
        self.lo, self.hi = lo, hi

    def quantize(self, col, w):
        q = np.clip(np.rint(w / self.scale), self.lo, self.hi)
        return q, self.scale * q


@pytest.mark.parametrize("clamp", [False, True])
@pytest.mark.parametrize("seed", range(10))
def test_equals_one_dimensional_row_major(seed, clamp):
    _, m, n, HL, HR, W, s = _problem(300 + seed)
    lo, hi = (-2, 1) if clamp else (None, None)
    res = g2.gptq2d_from_grams(W, HL, HR, s, lo, hi)
    U = go.inverse_factor(np.kron(HL, HR))
    grid = _ClampedGrid(s, lo, hi) if clamp else go.IntegerGrid(s)
    codes, deq, E = go.gptq_core(W.reshape(1, m * n), U, 1, grid)
    assert np.array_equal(codes.reshape(m, n), res["codes"])
    assert np.allclose(E.reshape(m, n), res["E"], rtol=1e-9, atol=1e-12)
    # the factor of the Kronecker Gram is the Kronecker product of the factors
    assert np.allclose(U, np.kron(res["UL"], res["UR"]), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("seed", range(10))
def test_equals_one_dimensional_column_major(seed):
    _, m, n, HL, HR, W, s = _problem(400 + seed)
    res = g2.gptq2d_from_grams(W, HL, HR, s)
    # column-major vec(W): Gram HR kron HL, entries visited column by column
    U = go.inverse_factor(np.kron(HR, HL))
    codes, deq, E = go.gptq_core(W.T.reshape(1, m * n), U, 1, go.IntegerGrid(s))
    assert np.array_equal(codes.reshape(n, m).T, res["codes"])
    assert np.allclose(E.reshape(n, m).T, res["E"], rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_equals_exact_sequential_minimisation(seed):
    rng = np.random.default_rng(500 + seed)
    m, n = int(rng.integers(2, 4)), int(rng.integers(2, 4))
    # small-denominator rational Grams (diagonally dominant, so positive definite)
    def gram(k):
        A = [[Fraction(int(rng.integers(-3, 4)), 8) for _ in range(k)] for _ in range(k)]
        return [[(A[i][j] + A[j][i]) / 2 + (2 if i == j else 0) for j in range(k)] for i in range(k)]
    HL, HR = gram(m), gram(n)
    W = [[Fraction(int(rng.integers(-40, 41)), 17) for _ in range(n)] for _ in range(m)]
    codes, decision = _sequential_exact(_kron_frac(HL, HR), [x for r in W for x in r])
    res = g2.gptq2d_from_grams(_fl(W), _fl(HL), _fl(HR))
    assert np.array_equal(res["codes"].reshape(-1), np.array(codes, dtype=np.float64))
    assert np.allclose(res["decision"].reshape(-1), [float(x) for x in decision], atol=1e-10)


# ---------------------------------------------------------------------------
# Babai, brute force and the error bound
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_reversed_order_is_babai_on_kronecker_lattice(seed):
    _, m, n, HL, HR, W, s = _problem(600 + seed, max_dim=4)
    # GPTQ run forward on vec(W) is Babai's nearest plane with the basis order
    # reversed: basis B with B^T B = J G J, target B J vec(W), codes J c.
    G = np.kron(HL, HR)
    J = np.arange(m * n)[::-1]
    Gr = G[np.ix_(J, J)]
    B = np.linalg.cholesky(Gr).T
    c, bstar2 = babai_nearest_plane(s * B, B @ W.reshape(-1)[J])
    babai_codes = np.zeros(m * n)
    babai_codes[J] = c
    res = g2.gptq2d_from_grams(W, HL, HR, s)
    assert np.array_equal(res["codes"].reshape(-1), babai_codes)
    loss = g2.two_sided_objective(W, res["deq"], HL, HR)
    assert loss <= 0.25 * np.sum(bstar2) * (1 + 1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_lower_bound(seed):
    rng = np.random.default_rng(700 + seed)
    m, n = 2, int(rng.integers(1, 4))
    HL, HR = _random_spd(rng, m, 8.0), _random_spd(rng, n, 8.0)
    W = rng.uniform(-1.5, 1.5, (m, n))
    res = g2.gptq2d_from_grams(W, HL, HR)
    base = np.floor(W).astype(int)
    best = np.inf
    for off in itertools.product(range(-1, 3), repeat=m * n):
        Q = base + np.array(off).reshape(m, n)
        best = min(best, g2.two_sided_objective(W, Q, HL, HR))
    assert g2.two_sided_objective(W, res["codes"], HL, HR) >= best - 1e-12


@pytest.mark.parametrize("seed", range(6))
def test_babai_error_bound(seed):
    _, m, n, HL, HR, W, s = _problem(800 + seed, max_dim=12)
    res = g2.gptq2d_from_grams(W, HL, HR, s)
    bound = 0.25 * s * s * np.sum(1.0 / np.outer(np.diag(res["UL"]), np.diag(res["UR"])) ** 2)
    assert g2.two_sided_objective(W, res["deq"], HL, HR) <= bound * (1 + 1e-12)


# ---------------------------------------------------------------------------
# closed forms and special cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("clamp", [False, True])
@pytest.mark.parametrize("seed", range(5))
def test_closed_forms(seed, clamp):
    rng = np.random.default_rng(900 + seed)
    m, n = int(rng.integers(5, 40)), int(rng.integers(5, 40))
    HL, HR = _random_spd(rng, m, 50.0), _random_spd(rng, n, 50.0)
    W = rng.standard_normal((m, n))
    lo, hi = (-1, 1) if clamp else (None, None)
    res = g2.gptq2d_from_grams(W, HL, HR, 0.5, lo, hi)
    UL, UR, E = res["UL"], res["UR"], res["E"]
    assert np.allclose(W - res["deq"], UL.T @ E @ UR, atol=1e-10)
    assert np.isclose(g2.two_sided_objective(W, res["deq"], HL, HR), np.sum(E * E), rtol=1e-9)
    # decision value = dequantized value + scaled error * UL_ii * UR_jj
    assert np.allclose(res["decision"], res["deq"] + E * np.outer(np.diag(UL), np.diag(UR)), atol=1e-12)
    if clamp:
        assert res["codes"].min() >= -1 and res["codes"].max() <= 1


@pytest.mark.parametrize("seed", range(4))
def test_identity_left_gram_is_one_sided_rows(seed):
    rng = np.random.default_rng(1000 + seed)
    m, n = int(rng.integers(1, 9)), int(rng.integers(1, 30))
    HR = _random_spd(rng, n, 40.0)
    W = rng.standard_normal((m, n))
    res = g2.gptq2d_from_grams(W, np.eye(m), HR, 0.25)
    codes, deq, E = go.gptq_core(W, go.inverse_factor(HR), 128, go.IntegerGrid(0.25))
    assert np.array_equal(res["codes"], codes)
    assert np.allclose(res["E"], E, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_identity_right_gram_is_one_sided_columns(seed):
    rng = np.random.default_rng(1100 + seed)
    m, n = int(rng.integers(1, 30)), int(rng.integers(1, 9))
    HL = _random_spd(rng, m, 40.0)
    W = rng.standard_normal((m, n))
    res = g2.gptq2d_from_grams(W, HL, np.eye(n), 0.25)
    codes, deq, E = go.gptq_core(W.T, go.inverse_factor(HL), 128, go.IntegerGrid(0.25))
    assert np.array_equal(res["codes"], codes.T)
    assert np.allclose(res["E"], E.T, atol=1e-12)


def test_diagonal_grams_give_round_to_nearest():
    rng = np.random.default_rng(1200)
    m, n = 7, 11
    HL = np.diag(rng.uniform(0.5, 3.0, m))
    HR = np.diag(rng.uniform(0.5, 3.0, n))
    W = rng.uniform(-4, 4, (m, n))
    res = g2.gptq2d_from_grams(W, HL, HR, 0.5, -5, 5)
    assert np.array_equal(res["codes"], np.clip(np.rint(W / 0.5), -5, 5))
    assert np.array_equal(res["decision"], W)


def test_antidiagonals_cover_each_entry_once():
    for m, n in [(1, 1), (1, 7), (6, 1), (3, 5), (5, 3), (4, 4)]:
        seen = np.zeros((m, n), dtype=int)
        for d in range(m + n - 1):
            ii = g2.antidiagonal(d, m, n)
            assert len(ii) > 0
            seen[ii, d - ii] += 1
        assert np.all(seen == 1)


def test_empty_and_invalid():
    c, dq, E, dec = g2.gptq2d(np.zeros((0, 3)), np.zeros((0, 0)), np.eye(3))
    assert c.shape == (0, 3)
    with pytest.raises(ValueError):
        g2.gptq2d(np.zeros((2, 3)), np.eye(3), np.eye(3))
    with pytest.raises(ValueError):
        g2.gptq2d(np.zeros((2, 2)), np.eye(2), np.eye(2), scale=0.0)


def test_replaying_own_codes_is_the_identity():
    rng = np.random.default_rng(1300)
    m, n = 17, 23
    HL, HR = _random_spd(rng, m), _random_spd(rng, n)
    W = rng.standard_normal((m, n))
    res = g2.gptq2d_from_grams(W, HL, HR, 0.3, -3, 2)
    c, dq, E, dec = g2.gptq2d(W, res["UL"], res["UR"], 0.3, -3, 2, forced=res["codes"])
    assert np.array_equal(c, res["codes"])
    assert np.array_equal(E, res["E"]) and np.array_equal(dec, res["decision"])
    # replaying a flipped code changes only the entries below and to the right
    F = res["codes"].copy()
    F[5, 7] += 1
    c2, _, E2, dec2 = g2.gptq2d(W, res["UL"], res["UR"], 0.3, forced=F)
    changed = np.argwhere(~np.isclose(dec2, res["decision"], rtol=0, atol=1e-13))
    assert len(changed) > 0
    assert np.all((changed[:, 0] >= 5) & (changed[:, 1] >= 7))
    assert np.array_equal(dec2[5, 7], res["decision"][5, 7])

