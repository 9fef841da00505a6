"""GPTQ-2D: two-sided adaptive rounding, plain fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only the tests, the repository's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with the
CUDA library and never imports it.

Source: the GPTQ-2D abstract on the "Daily Papers" page.  Adaptive rounding
(GPTQ, i.e. Babai's nearest plane) rounds a real matrix to integers under a
quadratic metric, one entry at a time in a fixed order, feeding every rounding
error forward through a triangular matrix.  The two-sided task puts a fixed
nonsingular basis on each side of the residual: minimise ||A (W - Q) B||_F^2
over integer Q.  Vectorising W turns the metric into one whose Gram matrix is a
Kronecker product, so the one-dimensional algorithm applies unchanged but costs
quartic time; GPTQ-2D gives the identical rounded matrix in cubic time by
rounding anti-diagonal by anti-diagonal, the entries of one anti-diagonal being
independent of each other.

Readings taken where the abstract is silent (repeated in the design notes):

* Gram matrices.  For W of shape m x n, HL = A^T A (m x m) and HR = B B^T
  (n x n).  Row-major vectorisation gives vec(A D B) = (A kron B^T) vec(D), so
  the one-dimensional metric is G = HL kron HR.  With HL = I the task falls
  apart into independent rows, each the familiar one-sided GPTQ problem with
  Hessian HR.
* Factors.  UL and UR are the upper factors with UL^T UL = HL^-1 and
  UR^T UR = HR^-1 (the same kind of factor as the one-sided column loop).  The
  upper factor of G^-1 is then UL kron UR (a Kronecker product of upper
  triangular matrices with positive diagonals is one, and the factor is unique).
  No damping is added: the Grams are taken as given, positive definite.
* Coupling.  The entry of UL kron UR that feeds the error of entry (i', j')
  into entry (i, j) is UL[i', i] * UR[j', j]; it vanishes unless i' <= i and
  j' <= j.  Entry (i, j) therefore sees exactly the errors of the entries above
  and to the left of it, all of which lie on earlier anti-diagonals, so every
  processing order that respects this partial order (row-major, column-major,
  anti-diagonal) rounds identically.
* Cubic form.  With M = E @ UR (E the scaled errors found so far, zero for
  entries not yet rounded), the current value of entry (i, j) is
  W[i, j] - sum_{i' <= i} UL[i', i] * M[i', j]; rounding entry (i, j) adds
  e_ij * UR[j, :] to row i of M.  Each anti-diagonal costs O(m n), i.e. the
  whole pass O(m n (m + n)).
* Grid.  The integers scaled by one positive scalar ``scale``, round half to
  even, optionally clamped to [qmin, qmax].  Clamping acts entry by entry, so it
  keeps the identity with the one-dimensional algorithm.
"""
from __future__ import annotations

import numpy as np

from .gptq_oracle import inverse_factor

__all__ = [
    "antidiagonal",
    "round_entries",
    "gptq2d",
    "gptq2d_from_grams",
    "two_sided_objective",
]


def antidiagonal(d, m, n):
    """Row indices i (ascending) of the entries (i, d - i) of an m x n matrix."""
    lo = max(0, d - (n - 1))
    hi = min(d, m - 1)
    return np.arange(lo, hi + 1)


def round_entries(v, scale, qmin=None, qmax=None):
    """Integer codes q = clamp(rint(v / scale), qmin, qmax) and scale * q."""
    q = np.rint(np.asarray(v, dtype=np.float64) / scale)
    if qmin is not None:
        q = np.maximum(q, qmin)
    if qmax is not None:
        q = np.minimum(q, qmax)
    return q, scale * q


def gptq2d(W, UL, UR, scale=1.0, qmin=None, qmax=None, forced=None):
    """Two-sided GPTQ, anti-diagonal by anti-diagonal (cubic form).

    W: [m, n]; UL: [m, m] and UR: [n, n] upper factors of HL^-1 and HR^-1.
    Returns (codes, deq, E, decision): the integer codes, scale * codes, the
    scaled errors e_ij = (wt_ij - scale * q_ij) / (UL_ii * UR_jj), and the
    values wt_ij the entries had when they were rounded.

    ``forced`` (an [m, n] array of integers) replays given codes instead of
    rounding: the feedback then follows those codes, and ``decision`` holds the
    values at which another implementation that chose them had to decide.
    """
    W = np.asarray(W, dtype=np.float64)
    UL = np.asarray(UL, dtype=np.float64)
    UR = np.asarray(UR, dtype=np.float64)
    m, n = W.shape
    if UL.shape != (m, m) or UR.shape != (n, n):
        raise ValueError("factor shapes do not match W")
    if not scale > 0:
        raise ValueError("scale must be positive")
    codes = np.zeros((m, n))
    deq = np.zeros((m, n))
    E = np.zeros((m, n))
    decision = np.zeros((m, n))
    M = np.zeros((m, n))  # M = E @ UR for the errors found so far
    for d in range(m + n - 1):
        ii = antidiagonal(d, m, n)
        jj = d - ii
        # current values: W[i, j] - sum_{i'} UL[i', i] * M[i', j]
        wt = W[ii, jj] - np.einsum("ki,ki->i", UL[:, ii], M[:, jj])
        q, dq = round_entries(wt, scale, qmin, qmax)
        if forced is not None:
            q = np.asarray(forced, dtype=np.float64)[ii, jj]
            dq = scale * q
        e = (wt - dq) / (UL[ii, ii] * UR[jj, jj])
        codes[ii, jj] = q
        deq[ii, jj] = dq
        E[ii, jj] = e
        decision[ii, jj] = wt
        M[ii, :] += e[:, None] * UR[jj, :]
    return codes, deq, E, decision


def gptq2d_from_grams(W, HL, HR, scale=1.0, qmin=None, qmax=None):
    """Factor the two Grams (UL^T UL = HL^-1, UR^T UR = HR^-1), then ``gptq2d``.

    Returns a dict with codes, deq, E, decision, UL and UR.
    """
    UL = inverse_factor(HL)
    UR = inverse_factor(HR)
    codes, deq, E, decision = gptq2d(W, UL, UR, scale, qmin, qmax)
    return {"codes": codes, "deq": deq, "E": E, "decision": decision, "UL": UL, "UR": UR}


def two_sided_objective(W, Q, HL, HR):
    """||A (W - Q) B||_F^2 written with the Grams: tr(HL D HR D^T), D = W - Q."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    return float(np.einsum("ab,bj,jk,ak->", np.asarray(HL, dtype=np.float64), D,
                           np.asarray(HR, dtype=np.float64), D))
