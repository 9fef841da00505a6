"""GPTQ per-layer quantization pass: plain, slow, fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only the tests, the repository's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with the
CUDA library (no kernels, headers, tables or helpers) and never imports it.

Sources (the method is stated in words only; each step below restates them):

* GPTQ knowledge note, "How It Works": for each linear layer the Hessian of the
  layer-output reconstruction loss is H = 2 X X^T, built from recorded layer
  inputs; after a column is quantized, inverse-Hessian information decides how
  the still-unquantized columns are adjusted.  All output rows follow one column
  order, 128-column blocks accumulate their corrections before one global
  update of the remaining matrix, and a damped Cholesky formulation supplies
  the (numerically stable) correction rows.
* GPTQ knowledge note, "Common Confusions": GPTQ and round-to-nearest share the
  same fixed low-bit grid; GPTQ only adds the error compensation.
* Encyclopedia article "GPTQ", "Technical Approach": 4/3/2-bit grids and
  group-wise quantization with one scale per group of weights.
* "Daily Papers" GPTQ-2D abstract: entries are processed in a fixed order, one
  at a time, each rounding error fed forward through a triangular matrix.
* "Daily Papers" GPTQ = Babai abstract: run back to front, GPTQ is Babai's
  nearest-plane algorithm on the lattice of H (used by the tests as a pin).
* Anthology record SOTA-185, "Filed as the approach, not the artifact" (the
  AWQ comparison): GPTQ has an optional reordering trick (act-order); the order
  used here is columns by descending diag(H).

Readings taken where the pages are silent (each is repeated in the design
notes of the repository):

* H is scaled by alpha = 2/N (N calibration tokens).  Every result below is
  invariant to a positive scale of H because damping is relative.
* damp is relative: lambda = damp * mean(diag H), added after dead columns
  (H_ii == 0) are set to H_ii = 1 and their weights to 0.
* Grid: asymmetric uniform min-max over the group, range widened to include 0;
  an all-zero group uses [0, 1] (scale 1/maxq, zero 0), which holds 0 exactly
  and keeps its zero-point off a rounding tie.  scale = (xmax - xmin) / maxq,
  zero = rint(-xmin / scale), code = clamp(rint(w / scale) + zero, 0, maxq),
  dequantized value = scale * (code - zero).  rint is round-half-to-even.
* Group parameters are fixed when the group's first column (in processing
  order) is reached, from the weights as updated so far.  group == 0 means one
  group per row, fixed from the row before any update.  Group size and block
  size must nest (one divides the other) so that the lazy blocks stay an exact
  reordering of the one-column-at-a-time procedure.
* Act-order: perm = stable argsort of -diag(H) (after the dead-column fix,
  before damping); groups are contiguous in processing order and g_idx maps an
  original column to its group.
* The upper factor U satisfies U^T U = (H + lambda I)^-1 (upper Cholesky factor
  of the damped inverse); the scaled error of column j is
  e_j = (w_j - dequant_j) / U_jj and the update of a later column k is
  w_k -= e_j * U_jk.

Every function here is pinned by a CPU test against values or properties that
do not come from this file (hand-derived worked examples, an independently
written Babai nearest-plane run, brute-force enumeration, closed-form
identities, special cases that reduce to round-to-nearest).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "NotPositiveDefinite",
    "hessian",
    "accumulate_hessian",
    "prepare",
    "inverse_factor",
    "inverse_factor_reversed",
    "group_params",
    "quantize_values",
    "group_params_f32",
    "quantize_values_f32",
    "MinMaxGrid",
    "IntegerGrid",
    "gptq_core",
    "gptq_quantize",
    "rtn_quantize",
    "rtn_quantize_f32",
    "gptq_layer",
    "layer_output_error",
    "pack_codes",
    "unpack_codes",
    "packed_words_per_row",
    "dequant_matvec",
]


class NotPositiveDefinite(ValueError):
    """The damped Hessian has no Cholesky factor (a pivot <= 0)."""


# ---------------------------------------------------------------------------
# Hessian (knowledge note "How It Works": H = 2 X X^T from recorded inputs)
# ---------------------------------------------------------------------------

def hessian(X, alpha=None):
    """H = alpha * X^T X in fp64 for token-major X of shape [N_tok, n].

    The pages write H = 2 X X^T with X stored features x tokens; the token-major
    array used here is its transpose, so the same product is X^T X.  alpha
    defaults to 2/N_tok.
    """
    X = np.asarray(X, dtype=np.float64)
    if alpha is None:
        alpha = 2.0 / max(X.shape[0], 1)
    return alpha * (X.T @ X)


def accumulate_hessian(H, X, alpha):
    """H + alpha * X^T X for one more token-major chunk X (fp64)."""
    X = np.asarray(X, dtype=np.float64)
    return np.asarray(H, dtype=np.float64) + alpha * (X.T @ X)


# ---------------------------------------------------------------------------
# Preprocessing: dead columns, damping, act-order
# (knowledge note "How It Works": "damped"; SOTA-185: the reordering trick)
# ---------------------------------------------------------------------------

def prepare(H, W, damp, act_order, diag=None):
    """Dead-column fix, relative damping and the optional act-order permutation.

    Returns a dict with
      H      damped Hessian in processing order (fp64 [n, n])
      W      weights with dead columns zeroed, in processing order (fp64)
      perm   processing position -> original column (int64 [n])
      dead   bool [n], original column order
      lam    the damping added to the diagonal

    ``diag`` optionally supplies the diagonal used for the dead-column test and
    the act-order key (the same values as diag(H), computed separately).
    """
    H = np.array(H, dtype=np.float64, copy=True)
    W = np.array(W, dtype=np.float64, copy=True)
    n = H.shape[0]
    if H.shape != (n, n) or W.shape[1] != n:
        raise ValueError("shape mismatch")
    key = np.diag(H).copy() if diag is None else np.array(diag, dtype=np.float64)
    dead = key == 0.0
    idx = np.flatnonzero(dead)
    H[idx, idx] = 1.0
    key[dead] = 1.0
    W[:, dead] = 0.0
    lam = float(damp) * float(np.mean(np.diag(H))) if n else 0.0
    if act_order:
        perm = np.argsort(-key, kind="stable")
    else:
        perm = np.arange(n)
    H[np.arange(n), np.arange(n)] += lam
    H = H[np.ix_(perm, perm)]
    W = W[:, perm]
    return {"H": H, "W": W, "perm": perm.astype(np.int64), "dead": dead, "lam": lam}


# ---------------------------------------------------------------------------
# Cholesky formulation of the inverse (knowledge note "How It Works")
# ---------------------------------------------------------------------------

def _cholesky(A):
    try:
        return np.linalg.cholesky(A)
    except np.linalg.LinAlgError as exc:  # a pivot <= 0
        raise NotPositiveDefinite(str(exc)) from exc


def _lower_inverse(L):
    import scipy.linalg

    return scipy.linalg.solve_triangular(L, np.eye(L.shape[0]), lower=True)


def inverse_factor(Hd):
    """Upper U with U^T U = Hd^-1, textbook three steps.

    1. Hd = L L^T (Cholesky), 2. Hd^-1 = L^-T L^-1, 3. U = upper Cholesky
    factor of Hd^-1.  U's rows are the correction rows of the column loop.
    """
    Hd = np.asarray(Hd, dtype=np.float64)
    if Hd.shape[0] == 0:
        return np.zeros((0, 0))
    L = _cholesky(Hd)
    Linv = _lower_inverse(L)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return _cholesky(Hinv).T


def inverse_factor_reversed(Hd):
    """Same U from one Cholesky and one triangular inverse.

    With J the order-reversal permutation, J Hd J = Lr Lr^T gives Hd = R R^T
    with R = J Lr J upper triangular, so U = R^-1 = J Lr^-1 J satisfies
    U^T U = Hd^-1 with a positive diagonal, i.e. it is the same factor as the
    three-step route (uniqueness of the Cholesky factor).
    """
    Hd = np.asarray(Hd, dtype=np.float64)
    if Hd.shape[0] == 0:
        return np.zeros((0, 0))
    Lr = _cholesky(Hd[::-1, ::-1])
    return _lower_inverse(Lr)[::-1, ::-1].copy()


# ---------------------------------------------------------------------------
# The grid (encyclopedia "Technical Approach": low-bit grid, one scale per group)
# ---------------------------------------------------------------------------

def group_params(cols, maxq):
    """Per-row (scale, zero) of the asymmetric min-max grid over ``cols`` [rows, g]."""
    cols = np.asarray(cols, dtype=np.float64)
    xmin = np.minimum(cols.min(axis=1), 0.0)
    xmax = np.maximum(cols.max(axis=1), 0.0)
    both = (xmin == 0.0) & (xmax == 0.0)
    xmax = np.where(both, 1.0, xmax)
    scale = (xmax - xmin) / maxq
    zero = np.rint(-xmin / scale)
    return scale, zero


def quantize_values(w, scale, zero, maxq):
    """codes = clamp(rint(w/scale) + zero, 0, maxq); dequant = scale*(code - zero)."""
    q = np.clip(np.rint(w / scale) + zero, 0.0, float(maxq))
    return q, scale * (q - zero)


def group_params_f32(cols, maxq):
    """The grid parameters evaluated step by step in IEEE float32.

    This is the bit-exactness reference for a float32 implementation of the
    same grid: every operation rounds to float32 once, in the order written.
    """
    cols = np.asarray(cols, dtype=np.float32)
    f0 = np.float32(0.0)
    xmin = np.minimum(cols.min(axis=1), f0)
    xmax = np.maximum(cols.max(axis=1), f0)
    both = (xmin == f0) & (xmax == f0)
    xmax = np.where(both, np.float32(1.0), xmax).astype(np.float32)
    scale = ((xmax - xmin).astype(np.float32) / np.float32(maxq)).astype(np.float32)
    zero = np.rint((-xmin).astype(np.float32) / scale).astype(np.float32)
    return scale, zero


def quantize_values_f32(w, scale, zero, maxq):
    """``quantize_values`` in float32, each operation rounded once."""
    w = np.asarray(w, dtype=np.float32)
    scale = np.asarray(scale, dtype=np.float32)
    zero = np.asarray(zero, dtype=np.float32)
    r = np.rint((w / scale).astype(np.float32)).astype(np.float32)
    q = np.clip((r + zero).astype(np.float32), np.float32(0.0), np.float32(maxq)).astype(np.float32)
    deq = (scale * (q - zero).astype(np.float32)).astype(np.float32)
    return q, deq


class MinMaxGrid:
    """Group-wise asymmetric min-max grid with parameters fixed at group start."""

    def __init__(self, rows, n, bits, group, block):
        if bits not in (2, 3, 4, 8):
            raise ValueError("bits must be 2, 3, 4 or 8")
        self.maxq = (1 << bits) - 1
        self.n = n
        self.G = group if group > 0 else max(n, 1)
        if group > 0 and not (block % group == 0 or group % block == 0):
            raise ValueError("group size and block size must nest")
        self.n_groups = -(-n // self.G) if n else 0
        self.scales = np.zeros((rows, self.n_groups))
        self.zeros = np.zeros((rows, self.n_groups))
        self._s = self._z = None

    def starts_group(self, col):
        return col % self.G == 0

    def group_end(self, col):
        return min(col + self.G, self.n)

    def set_params(self, col, cur):
        s, z = group_params(cur, self.maxq)
        g = col // self.G
        self.scales[:, g] = s
        self.zeros[:, g] = z
        self._s, self._z = s, z

    def quantize(self, col, w):
        return quantize_values(w, self._s, self._z, self.maxq)


class IntegerGrid:
    """Unbounded integer grid with a fixed scale (no clamp, no groups).

    Used by the worked examples and by the nearest-plane cross-check, where the
    lattice is the integer lattice scaled by ``scale``.
    """

    def __init__(self, scale=1.0):
        self.scale = float(scale)

    def starts_group(self, col):
        return False

    def group_end(self, col):  # pragma: no cover - never called
        return col + 1

    def set_params(self, col, cur):  # pragma: no cover - never called
        pass

    def quantize(self, col, w):
        q = np.rint(w / self.scale)
        return q, self.scale * q


# ---------------------------------------------------------------------------
# The column loop (knowledge note "How It Works"; GPTQ-2D abstract)
# ---------------------------------------------------------------------------

def gptq_core(W, U, block, grid):
    """Quantize the columns of W (already in processing order) one at a time.

    For each block [i1, i2) of ``block`` columns and each column j in it:
    fix the group parameters if a group starts at j, quantize the current
    value of column j, form the scaled error e_j = (w_j - dequant_j) / U_jj,
    and subtract e_j * U[j, k] from every later column k of the block.  After
    the block, the remaining columns receive the accumulated update
    W[:, i2:] -= E[:, i1:i2] @ U[i1:i2, i2:] in one matrix product.

    Returns (codes, dequant, E) in processing order; ``grid`` keeps the
    per-group scales and zeros.
    """
    W = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    rows, n = W.shape
    if block < 1:
        raise ValueError("block must be >= 1")
    codes = np.zeros((rows, n))
    deq = np.zeros((rows, n))
    E = np.zeros((rows, n))
    for i1 in range(0, n, block):
        i2 = min(i1 + block, n)
        Wb = W[:, i1:i2].copy()
        for j in range(i2 - i1):
            col = i1 + j
            if grid.starts_group(col):
                hi = grid.group_end(col)
                if hi > i2:
                    cur = np.concatenate([Wb[:, j:], W[:, i2:hi]], axis=1)
                else:
                    cur = Wb[:, j:hi - i1]
                grid.set_params(col, cur)
            q, dq = grid.quantize(col, Wb[:, j])
            e = (Wb[:, j] - dq) / U[col, col]
            Wb[:, j + 1:] -= np.outer(e, U[col, col + 1:i2])
            codes[:, col] = q
            deq[:, col] = dq
            E[:, col] = e
        W[:, i2:] -= E[:, i1:i2] @ U[i1:i2, i2:]
    return codes, deq, E


def gptq_quantize(W, U, bits, group, block):
    """GPTQ on the min-max grid; W and U already in processing order.

    Returns dict(codes, deq, E, scales, zeros) in processing order, with
    scales/zeros of shape [rows, n_groups] indexed by processing-order group.
    """
    W = np.asarray(W, dtype=np.float64)
    grid = MinMaxGrid(W.shape[0], W.shape[1], bits, group, block)
    codes, deq, E = gptq_core(W, U, block, grid)
    return {"codes": codes.astype(np.int64), "deq": deq, "E": E,
            "scales": grid.scales, "zeros": grid.zeros}


# ---------------------------------------------------------------------------
# Round-to-nearest baseline (knowledge note "Common Confusions", "Why It Exists")
# ---------------------------------------------------------------------------

def _rtn(W, bits, group, params, quant):
    rows, n = W.shape
    maxq = (1 << bits) - 1
    G = group if group > 0 else max(n, 1)
    ng = -(-n // G) if n else 0
    codes = np.zeros((rows, n))
    deq = np.zeros((rows, n), dtype=W.dtype)
    scales = np.zeros((rows, ng), dtype=W.dtype)
    zeros = np.zeros((rows, ng), dtype=W.dtype)
    for g in range(ng):
        c0, c1 = g * G, min((g + 1) * G, n)
        s, z = params(W[:, c0:c1], maxq)
        scales[:, g], zeros[:, g] = s, z
        for c in range(c0, c1):
            q, d = quant(W[:, c], s, z, maxq)
            codes[:, c], deq[:, c] = q, d
    return {"codes": codes.astype(np.int64), "deq": deq, "scales": scales, "zeros": zeros}


def rtn_quantize(W, bits, group):
    """Round-to-nearest on the same grid, groups of ``group`` original columns."""
    return _rtn(np.asarray(W, dtype=np.float64), bits, group, group_params, quantize_values)


def rtn_quantize_f32(W, bits, group):
    """Round-to-nearest with every grid operation in IEEE float32."""
    return _rtn(np.asarray(W, dtype=np.float32), bits, group, group_params_f32, quantize_values_f32)


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def gptq_layer(W, X=None, H=None, bits=4, group=128, damp=0.01, block=128,
               act_order=False, diag=None, factor="three_step"):
    """H (from X if not given) -> preprocessing -> U -> column loop -> outputs.

    Outputs in original column order: codes, deq (dequantized Q), g_idx.  In
    processing order: E, scales, zeros, perm.  Also U, the damped permuted H,
    the prepared W and row_loss = sum_j e_j^2 per row.
    """
    W = np.asarray(W, dtype=np.float64)
    if H is None:
        H = hessian(X)
    prep = prepare(H, W, damp, act_order, diag=diag)
    if factor == "three_step":
        U = inverse_factor(prep["H"])
    else:
        U = inverse_factor_reversed(prep["H"])
    res = gptq_quantize(prep["W"], U, bits, group, block)
    perm = prep["perm"]
    rows, n = W.shape
    codes = np.zeros((rows, n), dtype=np.int64)
    deq = np.zeros((rows, n))
    codes[:, perm] = res["codes"]
    deq[:, perm] = res["deq"]
    G = group if group > 0 else max(n, 1)
    g_idx = np.zeros(n, dtype=np.int64)
    g_idx[perm] = np.arange(n) // G
    return {
        "codes": codes, "deq": deq, "g_idx": g_idx, "perm": perm,
        "scales": res["scales"], "zeros": res["zeros"], "E": res["E"],
        "U": U, "H": prep["H"], "W": prep["W"], "dead": prep["dead"],
        "lam": prep["lam"], "row_loss": np.sum(res["E"] ** 2, axis=1),
    }


def layer_output_error(W, Q, S):
    """||(W - Q) X||_F^2 written as tr(D S D^T) with S = X^T X (undamped)."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    return float(np.einsum("ij,jk,ik->", D, np.asarray(S, dtype=np.float64), D))


# ---------------------------------------------------------------------------
# Packing (knowledge note "Tradeoffs": packed weights; encyclopedia
# "Performance and Accuracy": 4 bits is half a byte per weight)
# ---------------------------------------------------------------------------

def packed_words_per_row(n, bits):
    """Each run of 32 codes fills exactly ``bits`` 32-bit words."""
    return bits * (-(-n // 32))


def pack_codes(codes, bits):
    """Row bitstream: code j of a row occupies bits [j*bits, (j+1)*bits) of the
    row's little-endian sequence of 32-bit words; rows are padded with zero
    codes to a multiple of 32 codes."""
    codes = np.asarray(codes, dtype=np.int64)
    rows, n = codes.shape
    if np.any(codes < 0) or np.any(codes >= (1 << bits)):
        raise ValueError("code out of range")
    words = packed_words_per_row(n, bits)
    bitplanes = (codes[:, :, None] >> np.arange(bits)) & 1          # [rows, n, bits]
    stream = np.zeros((rows, words * 32), dtype=np.int64)
    stream[:, : n * bits] = bitplanes.reshape(rows, n * bits)
    stream = stream.reshape(rows, words, 32)
    packed = np.sum(stream << np.arange(32), axis=2)
    return packed.astype(np.uint32)


def unpack_codes(packed, n, bits):
    """Inverse of ``pack_codes``."""
    packed = np.asarray(packed, dtype=np.int64)
    rows, words = packed.shape
    stream = (packed[:, :, None] >> np.arange(32)) & 1               # [rows, words, 32]
    stream = stream.reshape(rows, words * 32)[:, : n * bits].reshape(rows, n, bits)
    return np.sum(stream << np.arange(bits), axis=2).astype(np.int64)


# ---------------------------------------------------------------------------
# Inference with the packed weights (GPTQ abstract on the "Daily Papers" page:
# the packed 3/4-bit weights run generative inference faster than FP16; GPTQ
# knowledge note, "Tradeoffs": deployment reads packed weights)
# ---------------------------------------------------------------------------

def dequant_matvec(packed, scales, zeros, n, bits, group, x, g_idx=None):
    """y[b, r] = sum_c Q[r, c] * x[b, c] for the dequantized weights
    Q[r, c] = scales[r, g(c)] * (code[r, c] - zeros[r, g(c)]), where the codes
    are read back from the packed rows (original column order) and g(c) is
    g_idx[c] when given (act-order) else c // group (group 0: one group per
    row).  x is [batch, n]; fp64 throughout."""
    codes = unpack_codes(packed, n, bits).astype(np.float64)
    rows = codes.shape[0]
    G = group if group > 0 else max(n, 1)
    g = np.asarray(g_idx, dtype=np.int64) if g_idx is not None else np.arange(n) // G
    s = np.asarray(scales, dtype=np.float64)[:, g]
    z = np.asarray(zeros, dtype=np.float64)[:, g]
    Q = s * (codes - z)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    return x @ Q.T
