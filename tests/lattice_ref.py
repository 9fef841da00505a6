"""Independent closest-vector references used to pin the oracle.

Nothing here calls the oracle.  ``babai_nearest_plane`` is Babai's nearest-plane
algorithm written from its textbook definition (classical Gram-Schmidt on an
explicit basis, coefficients chosen from the last basis vector to the first);
``brute_force_cvp`` enumerates a box of integer vectors.  The GPTQ = Babai
abstract on the "Daily Papers" page states that GPTQ run from the last column
to the first is exactly this algorithm on the lattice whose Gram matrix is H.
"""
import itertools

import numpy as np


def gram_schmidt(B):
    """Classical Gram-Schmidt on the columns b_1..b_n of B (no normalisation)."""
    n = B.shape[1]
    Bs = np.zeros_like(B, dtype=np.float64)
    for i in range(n):
        v = B[:, i].astype(np.float64).copy()
        for k in range(i):
            mu = np.dot(B[:, i], Bs[:, k]) / np.dot(Bs[:, k], Bs[:, k])
            v -= mu * Bs[:, k]
        Bs[:, i] = v
    return Bs


def babai_nearest_plane(B, t):
    """Integer coefficients c with B c close to target t (Babai, nearest plane).

    For i = n..1: c_i = round(<t, b*_i> / <b*_i, b*_i>), then t <- t - c_i b_i.
    Returns (c, ||b*_i||^2 for all i).
    """
    Bs = gram_schmidt(B)
    n = B.shape[1]
    t = np.array(t, dtype=np.float64, copy=True)
    c = np.zeros(n)
    for i in range(n - 1, -1, -1):
        c[i] = np.rint(np.dot(t, Bs[:, i]) / np.dot(Bs[:, i], Bs[:, i]))
        t -= c[i] * B[:, i]
    return c, np.sum(Bs * Bs, axis=0)


def quad_loss(H, w, q):
    d = np.asarray(w, dtype=np.float64) - np.asarray(q, dtype=np.float64)
    return float(d @ np.asarray(H, dtype=np.float64) @ d)


def brute_force_cvp(H, w, radius=2):
    """Minimise (w-q)^T H (w-q) over integer q in a box around w."""
    w = np.asarray(w, dtype=np.float64)
    lo = np.floor(w).astype(int) - radius
    hi = np.ceil(w).astype(int) + radius
    best, best_q = np.inf, None
    for q in itertools.product(*[range(a, b + 1) for a, b in zip(lo, hi)]):
        val = quad_loss(H, w, q)
        if val < best:
            best, best_q = val, np.array(q, dtype=np.float64)
    return best_q, best
