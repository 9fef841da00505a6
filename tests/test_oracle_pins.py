"""Pins for the fp64 oracle: values and properties that do not come from it.

* hand-derived worked examples (tests/golden/worked_examples.json), exact fractions;
* hand-derived grid and packing examples (tests/golden/grid_examples.json, pack_examples.json);
* Babai's nearest plane, written independently in tests/lattice_ref.py (the
  GPTQ = Babai abstract on the "Daily Papers" page);
* brute-force closest vectors on tiny inputs;
* closed forms: U^T U H = I, W - Q = E U, sum e^2 = (w-q)^T H (w-q);
* special cases: diagonal H gives round-to-nearest (GPTQ knowledge note,
  "Common Confusions"); block size does not change the result ("How It Works":
  the lazy blocks only batch the corrections); a positive scale of H does not
  change it (damping is relative).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import gptq_oracle as go
from tests.lattice_ref import babai_nearest_plane, brute_force_cvp, quad_loss


def _frac_matrix(rows):
    return [[Fraction(x) for x in r] for r in rows]


def _exact_loss(H, w, q):
    n = len(w)
    d = [w[i] - q[i] for i in range(n)]
    return sum(d[i] * H[i][j] * d[j] for i in range(n) for j in range(n))


def _run_integer_gptq(H, w, order, block):
    H = np.asarray(H, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    perm = np.asarray(order)
    Hp = H[np.ix_(perm, perm)]
    U = go.inverse_factor(Hp)
    codes, deq, E = go.gptq_core(w[perm][None, :], U, block, go.IntegerGrid(1.0))
    decision = deq[0] + E[0] * np.diag(U)
    out = np.zeros(len(w))
    out[perm] = codes[0]
    return out, decision, E[0], U


# ---------------------------------------------------------------------------
# worked examples
# ---------------------------------------------------------------------------

def _cases(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("block", [1, 2, 128])
def test_worked_examples(golden_dir, block):
    for case in _cases(golden_dir, "worked_examples.json")["cases"]:
        Hq = _frac_matrix(case["H"])
        wq = [Fraction(x) for x in case["w"]]
        Hf = np.array([[float(x) for x in r] for r in Hq])
        wf = np.array([float(x) for x in wq])
        # golden losses are consistent with the golden codes (exact arithmetic)
        assert _exact_loss(Hq, wq, case["rtn_codes"]) == Fraction(case["rtn_loss"])
        for key in ("forward", "backward"):
            g = case[key]
            assert _exact_loss(Hq, wq, g["codes"]) == Fraction(g["loss"]), (case["name"], key)
            codes, decision, E, U = _run_integer_gptq(Hf, wf, g["order"], block)
            assert codes.tolist() == g["codes"], (case["name"], key)
            want = np.array([float(Fraction(x)) for x in g["decision_values"]])
            np.testing.assert_allclose(decision, want, rtol=0, atol=1e-12)
            # loss identity on the integer grid
            assert np.isclose(np.sum(E ** 2), float(Fraction(g["loss"])), rtol=1e-12)
        # round to nearest = rint of each weight (the shared grid)
        assert np.rint(wf).tolist() == case["rtn_codes"]
        # the optimum by enumeration
        q_opt, best = brute_force_cvp(Hf, wf, radius=2)
        assert q_opt.tolist() == case["optimum"]["codes"]
        assert np.isclose(best, float(Fraction(case["optimum"]["loss"])), rtol=1e-12)


def test_grid_examples(golden_dir):
    d = _cases(golden_dir, "grid_examples.json")
    for case in d["cases"]:
        maxq = (1 << case["bits"]) - 1
        w = np.array(case["w"])[None, :]
        s, z = go.group_params(w, maxq)
        assert np.isclose(s[0], case["scale"], rtol=1e-15, atol=0)
        assert z[0] == case["zero"]
        q, dq = go.quantize_values(w[0], s[0], z[0], maxq)
        assert q.tolist() == case["codes"], case["name"]
        np.testing.assert_allclose(dq, case["deq"], rtol=1e-15, atol=1e-16)
        # the float32 grid agrees on these (values chosen off rounding boundaries)
        s32, z32 = go.group_params_f32(w, maxq)
        q32, _ = go.quantize_values_f32(w[0], s32[0], z32[0], maxq)
        assert q32.tolist() == case["codes"], case["name"]
    c = d["clamp"]
    maxq = (1 << c["bits"]) - 1
    q, _ = go.quantize_values(np.array(c["w"]), c["scale"], c["zero"], maxq)
    assert q.tolist() == c["codes"]


def test_pack_examples(golden_dir):
    for case in _cases(golden_dir, "pack_examples.json")["cases"]:
        codes = np.array([case["codes"]])
        packed = go.pack_codes(codes, case["bits"])
        want = np.array([[int(x, 16) if x.startswith("0x") else int(x) for x in case["words"]]], dtype=np.uint32)
        assert packed.shape == want.shape, case["name"]
        assert np.array_equal(packed, want), (case["name"], [hex(x) for x in packed[0]])
        assert np.array_equal(go.unpack_codes(packed, codes.shape[1], case["bits"]), codes)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("n", [1, 31, 32, 33, 100])
def test_pack_roundtrip(bits, n):
    rng = np.random.default_rng(bits * 1000 + n)
    codes = rng.integers(0, 1 << bits, size=(3, n))
    packed = go.pack_codes(codes, bits)
    assert packed.shape == (3, go.packed_words_per_row(n, bits))
    assert np.array_equal(go.unpack_codes(packed, n, bits), codes)
    # bits per weight: a full run of 32 codes takes exactly `bits` words
    assert go.packed_words_per_row(32 * 7, bits) * 32 == 32 * 7 * bits


def test_dequant_matvec_examples(golden_dir):
    """Hand-derived packed matvec cases, natural groups and an act-order g_idx."""
    for case in _cases(golden_dir, "matvec_examples.json")["cases"]:
        packed = np.array([[int(w, 16) for w in row] for row in case["packed"]], dtype=np.uint32)
        y = go.dequant_matvec(packed, np.array(case["scales"]), np.array(case["zeros"]), case["n"], case["bits"],
                              case["group"], np.array(case["x"]), case.get("g_idx"))
        assert np.array_equal(y, np.array(case["y"]))


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("bits,group", [(4, 32), (3, 0), (2, 16)])
def test_dequant_matvec_matches_layer_dequantized_weights(act_order, bits, group):
    """Reading the codes back from the packed stream and applying the grid per
    g_idx reproduces the column loop's own dequantized weights (computed along
    a different path, inside the loop), so the matvec equals deq @ x."""
    rng = np.random.default_rng(3 + bits)
    rows, n = 5, 64
    X = rng.standard_normal((200, n)) * np.exp(rng.standard_normal(n))
    W = rng.standard_normal((rows, n)) * 0.02
    ref = go.gptq_layer(W, X=X, bits=bits, group=group, block=32, act_order=act_order)
    x = rng.standard_normal((3, n))
    y = go.dequant_matvec(go.pack_codes(ref["codes"], bits), ref["scales"], ref["zeros"], n, bits, group, x,
                          ref["g_idx"] if act_order else None)
    np.testing.assert_allclose(y, x @ ref["deq"].T, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# Hessian
# ---------------------------------------------------------------------------

def test_hessian_properties():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((300, 17))
    H = go.hessian(X)
    N = X.shape[0]
    assert np.allclose(H, H.T)
    for _ in range(5):
        v = rng.standard_normal(17)
        assert np.isclose(v @ H @ v, 2.0 / N * np.sum((X @ v) ** 2), rtol=1e-12)
    assert np.isclose(np.trace(H), 2.0 / N * np.sum(X * X), rtol=1e-12)
    # entries by a plain loop over tokens on a tiny case
    Xs = X[:7, :4]
    Hs = go.hessian(Xs, alpha=1.0)
    for i in range(4):
        for j in range(4):
            assert np.isclose(Hs[i, j], sum(Xs[t, i] * Xs[t, j] for t in range(7)), rtol=1e-13)
    # accumulating chunks equals one pass
    Hc = np.zeros((17, 17))
    for a in range(0, N, 64):
        Hc = go.accumulate_hessian(Hc, X[a:a + 64], 2.0 / N)
    assert np.allclose(Hc, H, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# inverse factor
# ---------------------------------------------------------------------------

def _random_spd(rng, n, cond=50.0):
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    ev = np.exp(rng.uniform(0, np.log(cond), n))
    return (Q * ev) @ Q.T


@pytest.mark.parametrize("n", [1, 2, 5, 33, 130])
def test_inverse_factor(n):
    rng = np.random.default_rng(n)
    H = _random_spd(rng, n)
    U = go.inverse_factor(H)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U @ H, np.eye(n), atol=1e-10)
    U2 = go.inverse_factor_reversed(H)
    assert np.allclose(U2, U, rtol=1e-10, atol=1e-12 * np.abs(U).max())


def test_inverse_factor_diagonal_and_damping():
    d = np.array([4.0, 1.0, 0.25, 9.0])
    U = go.inverse_factor(np.diag(d))
    assert np.allclose(U, np.diag(1.0 / np.sqrt(d)))
    # damping: H = I with damp 0.5 gives H' = 1.5 I, so U = I / sqrt(1.5)
    prep = go.prepare(np.eye(3), np.zeros((2, 3)), 0.5, False)
    assert np.isclose(prep["lam"], 0.5)
    assert np.allclose(go.inverse_factor(prep["H"]), np.eye(3) / np.sqrt(1.5))


def test_not_positive_definite():
    X = np.random.default_rng(0).standard_normal((3, 8))  # rank 3 < 8
    H = go.hessian(X)
    prep = go.prepare(H, np.zeros((1, 8)), 0.0, False)
    with pytest.raises(go.NotPositiveDefinite):
        go.inverse_factor(prep["H"])


# ---------------------------------------------------------------------------
# Babai and brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(8))
def test_back_to_front_is_babai(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 13))
    H = _random_spd(rng, n, cond=30.0)
    s = float(rng.uniform(0.2, 1.0))
    w = rng.standard_normal(n)
    # GPTQ from the last column to the first on the integer grid scaled by s
    perm = np.arange(n)[::-1]
    Hp = H[np.ix_(perm, perm)]
    U = go.inverse_factor(Hp)
    codes, deq, E = go.gptq_core(w[perm][None, :], U, 128, go.IntegerGrid(s))
    gptq_codes = np.zeros(n)
    gptq_codes[perm] = codes[0]
    # Babai on the lattice s * B Z^n with B^T B = H, target B w
    B = np.linalg.cholesky(H).T
    c, bstar2 = babai_nearest_plane(s * B, B @ w)
    assert np.array_equal(gptq_codes, c)
    loss = quad_loss(H, w, s * c)
    assert np.isclose(np.sum(E ** 2), loss, rtol=1e-9)
    # Babai's bound without clipping: error <= (1/4) sum ||b*_i||^2
    assert loss <= 0.25 * np.sum(bstar2) * (1 + 1e-12)
    assert np.isclose(0.25 * np.sum(bstar2), 0.25 * s * s * np.sum(1.0 / np.diag(U) ** 2), rtol=1e-9)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_lower_bound(seed):
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(2, 6))
    H = _random_spd(rng, n, cond=20.0)
    w = rng.uniform(-2, 2, n)
    U = go.inverse_factor(H)
    codes, deq, E = go.gptq_core(w[None, :], U, 128, go.IntegerGrid(1.0))
    _, best = brute_force_cvp(H, w, radius=2)
    assert quad_loss(H, w, codes[0]) >= best - 1e-12


# ---------------------------------------------------------------------------
# special cases and closed forms on the min-max grid
# ---------------------------------------------------------------------------

def _layer_inputs(seed, rows=24, n=96, tokens=400):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((tokens, n)) * np.exp(rng.standard_normal(n))[None, :]
    W = 0.02 * rng.standard_normal((rows, n))
    return W, X


@pytest.mark.parametrize("bits,group", [(4, 0), (3, 32), (2, 16), (8, 48), (4, 96)])
def test_diagonal_hessian_is_rtn(bits, group):
    rng = np.random.default_rng(bits + group)
    W = 0.02 * rng.standard_normal((10, 96))
    d = rng.uniform(0.5, 2.0, 96)
    block = 96 if group in (0, 48, 96) else 32
    out = go.gptq_layer(W, H=np.diag(d), bits=bits, group=group, damp=0.01, block=block)
    ref = go.rtn_quantize(W, bits, group)
    assert np.array_equal(out["codes"], ref["codes"])
    assert np.array_equal(out["scales"], ref["scales"])
    assert np.array_equal(out["zeros"], ref["zeros"])
    # with act-order the groups follow processing order: RTN of the permuted W
    out = go.gptq_layer(W, H=np.diag(d), bits=bits, group=group, damp=0.01, block=block, act_order=True)
    perm = out["perm"]
    assert np.array_equal(perm, np.argsort(-d, kind="stable"))
    ref = go.rtn_quantize(W[:, perm], bits, group)
    assert np.array_equal(out["codes"][:, perm], ref["codes"])
    assert np.array_equal(out["scales"], ref["scales"])


@pytest.mark.parametrize("group", [0, 16, 32, 64])
def test_block_size_does_not_change_result(group):
    W, X = _layer_inputs(7)
    base = None
    for block in (1, 16, 32, 64, 128):
        if group and not (block % group == 0 or group % block == 0):
            continue
        out = go.gptq_layer(W, X=X, bits=3, group=group, damp=0.01, block=block)
        if base is None:
            base = out
            continue
        assert np.array_equal(out["codes"], base["codes"]), block
        assert np.allclose(out["scales"], base["scales"], rtol=1e-12)
        assert np.allclose(out["E"], base["E"], rtol=1e-9, atol=1e-12)


def test_hessian_scale_invariance():
    W, X = _layer_inputs(8)
    H = go.hessian(X)
    a = go.gptq_layer(W, H=H, bits=4, group=32, damp=0.01, block=32)
    b = go.gptq_layer(W, H=37.5 * H, bits=4, group=32, damp=0.01, block=32)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["scales"], b["scales"], rtol=1e-12)


@pytest.mark.parametrize("act_order", [False, True])
def test_closed_form_identities(act_order):
    W, X = _layer_inputs(9)
    out = go.gptq_layer(W, X=X, bits=3, group=32, damp=0.01, block=32, act_order=act_order)
    Wp, U, E, Hd = out["W"], out["U"], out["E"], out["H"]
    perm = out["perm"]
    Qp = out["deq"][:, perm]
    # W - Q = E U (processing order)
    assert np.allclose(Wp - Qp, E @ U, atol=1e-12)
    # per-row loss identity
    D = Wp - Qp
    lhs = np.einsum("ij,jk,ik->i", D, Hd, D)
    assert np.allclose(lhs, out["row_loss"], rtol=1e-9)
    # group parameters come from the weights as updated when the group starts
    G = 32
    for g in range(W.shape[1] // G):
        c = g * G
        cur = Wp[:, c:c + G] - E[:, :c] @ U[:c, c:c + G]
        s, z = go.group_params(cur, 7)
        assert np.allclose(out["scales"][:, g], s, rtol=1e-12)
        assert np.array_equal(out["zeros"][:, g], z)


def test_act_order_equals_prepermuted_inputs():
    W, X = _layer_inputs(10)
    H = go.hessian(X)
    out = go.gptq_layer(W, H=H, bits=4, group=16, damp=0.01, block=32, act_order=True)
    perm = np.argsort(-np.diag(H), kind="stable")
    assert np.array_equal(out["perm"], perm)
    ref = go.gptq_layer(W[:, perm], H=H[np.ix_(perm, perm)], bits=4, group=16, damp=0.01, block=32)
    assert np.array_equal(out["codes"][:, perm], ref["codes"])
    assert np.array_equal(out["g_idx"][perm], np.arange(W.shape[1]) // 16)
    assert np.allclose(out["scales"], ref["scales"])


def test_dead_columns():
    W, X = _layer_inputs(11, n=64)
    X[:, [3, 40]] = 0.0
    out = go.gptq_layer(W, X=X, bits=4, group=32, damp=0.01, block=32)
    assert out["dead"][[3, 40]].all() and out["dead"].sum() == 2
    assert np.all(out["W"][:, [3, 40]] == 0.0)
    assert np.all(out["deq"][:, [3, 40]] == 0.0)
    H = go.hessian(X)
    assert np.isclose(out["H"][3, 3], 1.0 + out["lam"])
    assert np.isclose(out["lam"], 0.01 * np.mean(np.where(np.diag(H) == 0, 1.0, np.diag(H))))


def test_layer_output_error_formula():
    W, X = _layer_inputs(12, n=32, tokens=50)
    out = go.gptq_layer(W, X=X, bits=4, group=0, damp=0.01, block=32)
    S = X.T @ X
    direct = np.sum((X @ (W - out["deq"]).T) ** 2)
    assert np.isclose(go.layer_output_error(W, out["deq"], S), direct, rtol=1e-12)
    # GPTQ beats round-to-nearest on output error for correlated inputs (sanity, not an invariant)
    rtn = go.rtn_quantize(W, 4, 0)
    assert go.layer_output_error(W, out["deq"], S) < go.layer_output_error(W, rtn["deq"], S)


def test_rtn_f32_close_to_fp64():
    rng = np.random.default_rng(13)
    W = 0.02 * rng.standard_normal((64, 256))
    a = go.rtn_quantize(W, 4, 128)
    b = go.rtn_quantize_f32(W.astype(np.float32), 4, 128)
    assert np.mean(a["codes"] == b["codes"]) > 0.999
    assert np.allclose(a["scales"], b["scales"], rtol=1e-6)


def test_block_group_must_nest():
    with pytest.raises(ValueError):
        go.gptq_layer(np.zeros((2, 96)), H=np.eye(96), bits=4, group=48, block=32)


def test_public_names():
    for name in oracle.__all__ if hasattr(oracle, "__all__") else []:
        assert hasattr(oracle, name)
