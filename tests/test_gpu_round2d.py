"""GPTQ-2D on the GPU (gptq2d_round) against the fp64 oracle.

Rounding decides integers from floating-point values, and the kernel forms each
value in fp32 while the oracle uses fp64, so a value within a few fp32 ulps of a
rounding tie may legitimately round either way, after which the two runs feed
different errors forward.  The parity check therefore replays the GPU's own
codes through the oracle (fp64, same inputs): every GPU code must be a correct
rounding of the value the oracle computes for it from the GPU's earlier
decisions, up to TOL grid steps from a tie; the GPU's scaled errors must match
the replay's; and the closed form W - scale * Q = UL^T E UR must hold on the
GPU's outputs.  Codes must also agree with the oracle's own free run on nearly
every entry.

TOL: the value v_ij is W_ij minus a sum of at most m * n fp32 products formed
as two nested sums of length <= max(m, n); with the test's Grams (condition
number 30) the partial sums stay within ~100 grid steps, so fp32 rounding moves
v by < 100 * 4096 * 2^-24 ~ 2.5e-2 grid steps in the worst case and ~1e-4 in
practice; TOL = 2e-3 is far above the practical error and far below the 0.5
that a wrong decision is off by.
"""
import numpy as np
import pytest
import torch

from oracle import gptq2d_oracle as g2
from oracle import gptq_oracle as go

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq

TOL = 2e-3


def _spd(rng, k, cond):
    Q, _ = np.linalg.qr(rng.standard_normal((k, k)))
    return (Q * np.geomspace(1.0, cond, k)) @ Q.T


def _inputs(seed, m, n, cond=30.0):
    rng = np.random.default_rng(seed)
    # the binding takes row-major (C-contiguous) factors; the oracle's factor
    # is a transposed view, so copy it into row-major order
    UL = np.ascontiguousarray(go.inverse_factor(_spd(rng, m, cond)), dtype=np.float32)
    UR = np.ascontiguousarray(go.inverse_factor(_spd(rng, n, cond)), dtype=np.float32)
    W = rng.standard_normal((m, n)).astype(np.float32)
    return W, UL, UR


def _run(W, UL, UR, scale, clamp, wdtype=torch.float32, garbage_below=True):
    dev = "cuda"
    ULd, URd = UL.copy(), UR.copy()
    if garbage_below:  # the kernel must never read below the diagonals
        ULd[np.tril_indices_from(ULd, -1)] = np.nan
        URd[np.tril_indices_from(URd, -1)] = np.nan
    lo, hi = clamp if clamp else (None, None)
    out = gq.gptq2d_round(torch.tensor(W, device=dev).to(wdtype), torch.tensor(ULd, device=dev),
                          torch.tensor(URd, device=dev), scale, lo, hi)
    torch.cuda.synchronize()
    return out["codes"].cpu().numpy().astype(np.float64), out["E"].cpu().numpy().astype(np.float64)


def _admissible(codes, value, scale, clamp):
    r = value / scale
    q_lo, q_hi = np.rint(r - TOL), np.rint(r + TOL)
    if clamp:
        q_lo, q_hi = np.clip(q_lo, *clamp), np.clip(q_hi, *clamp)
    return (codes >= q_lo) & (codes <= q_hi)


def _check(W, UL, UR, scale, clamp, codes, E):
    W64, UL64, UR64 = W.astype(np.float64), UL.astype(np.float64), UR.astype(np.float64)
    lo, hi = clamp if clamp else (None, None)
    _, _, E_rep, dec = g2.gptq2d(W64, UL64, UR64, scale, lo, hi, forced=codes)
    ok = _admissible(codes, dec, scale, clamp)
    assert ok.all(), f"{np.count_nonzero(~ok)} wrong decisions, first at {np.argwhere(~ok)[0]}"
    assert np.abs(E - E_rep).max() <= 1e-3 * (np.abs(E_rep).max() + 1e-30)
    resid = W64 - scale * codes - UL64.T @ E @ UR64
    assert np.abs(resid).max() <= 1e-3 * (np.abs(W64).max() + scale)
    free, _, _, _ = g2.gptq2d(W64, UL64, UR64, scale, lo, hi)
    assert np.mean(free == codes) >= 0.99


SIZES = [(1, 1), (1, 70), (70, 1), (64, 64), (65, 130), (130, 65), (200, 333), (333, 200)]


@pytest.mark.parametrize("m,n", SIZES)
def test_round2d_parity(m, n):
    W, UL, UR = _inputs(10 + m + 7 * n, m, n)
    codes, E = _run(W, UL, UR, 0.25, None)
    _check(W, UL, UR, 0.25, None, codes, E)


@pytest.mark.parametrize("m,n", [(64, 64), (200, 333)])
def test_round2d_clamped(m, n):
    W, UL, UR = _inputs(20 + m, m, n)
    codes, E = _run(W, UL, UR, 0.25, (-4, 3))
    assert codes.min() >= -4 and codes.max() <= 3
    _check(W, UL, UR, 0.25, (-4, 3), codes, E)


def test_round2d_bf16_weights():
    W, UL, UR = _inputs(30, 150, 140)
    Wb = torch.tensor(W).to(torch.bfloat16).float().numpy()
    codes, E = _run(Wb, UL, UR, 0.25, None, wdtype=torch.bfloat16)
    _check(Wb, UL, UR, 0.25, None, codes, E)


def test_round2d_identity_left_gram_is_row_wise_gptq():
    # HL = I: every row is the one-sided problem with Hessian HR (integer grid)
    W, _, UR = _inputs(40, 96, 200)
    UL = np.eye(96, dtype=np.float32)
    codes, E = _run(W, UL, UR, 0.25, None)
    _check(W, UL, UR, 0.25, None, codes, E)
    ref, _, E1 = go.gptq_core(W.astype(np.float64), UR.astype(np.float64), 1, go.IntegerGrid(0.25))
    assert np.mean(ref == codes) >= 0.99


def test_round2d_deterministic():
    W, UL, UR = _inputs(50, 200, 260)
    a = _run(W, UL, UR, 0.25, None)
    b = _run(W, UL, UR, 0.25, None)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_round2d_without_error_output():
    # E = NULL: the errors live in the workspace; the codes are the same
    W, UL, UR = _inputs(60, 130, 190)
    dev = "cuda"
    args = (torch.tensor(W, device=dev), torch.tensor(UL, device=dev), torch.tensor(UR, device=dev), 0.25)
    a = gq.gptq2d_round(*args)
    b = gq.gptq2d_round(*args, want_E=False)
    torch.cuda.synchronize()
    assert b["E"] is None
    assert torch.equal(a["codes"], b["codes"])


def test_round2d_full_size_sampled():
    """W 4096 x 4096 (N(0, 0.02)), a 4-bit signed grid (scale 0.005, codes in
    [-8, 7]); HL and HR are Grams of 8192 N(0, 1) tokens built and factored by
    the library (damp 0.01).  Sampled entries: the value each one was rounded
    at, recomputed in fp64 from the GPU's errors of all entries above and to
    its left, must round to the GPU's code; the closed form holds there too."""
    m = n = 4096
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(4096)
    Hs = []
    for _ in range(2):
        X = torch.randn((8192, m), generator=g, device=dev).to(torch.bfloat16)
        H = torch.zeros((m, m), dtype=torch.float32, device=dev)
        gq.gptq_hessian_accum(H, X, 2.0 / 8192)
        Hs.append(H)
        del X
    UL = gq.gptq2d_factor(Hs[0], damp=0.01)
    UR = gq.gptq2d_factor(Hs[1], damp=0.01)
    W = 0.02 * torch.randn((m, n), generator=g, device=dev)
    out = gq.gptq2d_round(W, UL, UR, 0.005, -8, 7)
    torch.cuda.synchronize()
    codes = out["codes"].cpu().numpy().astype(np.float64)
    E = out["E"].cpu().numpy().astype(np.float64)
    Wh = W.cpu().numpy().astype(np.float64)
    ULh = UL.cpu().numpy().astype(np.float64)
    URh = UR.cpu().numpy().astype(np.float64)
    assert codes.min() >= -8 and codes.max() <= 7
    rng = np.random.default_rng(7)
    picks = [(0, 0), (m - 1, n - 1), (0, n - 1), (m - 1, 0)] + [tuple(x) for x in rng.integers(0, m, (44, 2))]
    for i, j in picks:
        full = ULh[: i + 1, i] @ (E[: i + 1, : j + 1] @ URh[: j + 1, j])
        own = ULh[i, i] * E[i, j] * URh[j, j]
        v = Wh[i, j] - (full - own)
        assert _admissible(np.array(codes[i, j]), np.array(v), 0.005, (-8, 7)), (i, j, v / 0.005, codes[i, j])
        e = (v - 0.005 * codes[i, j]) / (ULh[i, i] * URh[j, j])
        assert abs(e - E[i, j]) <= 1e-3 * 0.005 / (ULh[i, i] * URh[j, j]) + 1e-6 * abs(e)
