"""Precision of the lazy trailing update, studied on the CPU.

The column loop's trailing update W[:, i2:] -= E[:, i1:i2] U[i1:i2, i2:] runs
on the tensor cores; this module asks how exact that product must be for the
integer codes to stay those of the fp64 oracle.  It runs the column loop in
float32 (the GPU's in-block arithmetic, with the oracle's float32 grid) and
forms each trailing product under one of these models, every product summed
exactly and rounded once to float32 (the accumulator's own rounding is not
modelled):

  fp32     the exact product of the fp32 operands
  3xtf32   E_hi U_hi + E_hi U_lo + E_lo U_hi, x_hi = x with its 13 low
           mantissa bits cleared, x_lo = x - x_hi read as tf32 (its own low
           bits cleared too) - what the trailing kernel computes
  3xbf16   the same split with bf16 halves (x_hi = bf16(x), x_lo =
           bf16(x - x_hi), round to nearest even): half the tensor-core time
  tf32     E_hi U_hi alone
  bf16     bf16(E) bf16(U) alone

and reports the share of codes equal to the oracle's.  It imports the oracle
(this is test code) and shares nothing with the CUDA path.
"""
import numpy as np

from oracle import gptq_oracle as go


def _tf32(x):
    x = np.asarray(x, dtype=np.float32)
    return (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def _bf16(x):
    x = np.asarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def product(E, U, model):
    """E @ U (float32 operands) under one of the models above, as float32."""
    E = np.asarray(E, dtype=np.float32)
    U = np.asarray(U, dtype=np.float32)
    d = lambda a: a.astype(np.float64)
    if model == "fp32":
        p = d(E) @ d(U)
    elif model == "3xtf32":
        eh, uh = _tf32(E), _tf32(U)
        el, ul = _tf32(E - eh), _tf32(U - uh)
        p = d(eh) @ d(uh) + d(eh) @ d(ul) + d(el) @ d(uh)
    elif model == "3xbf16":
        eh, uh = _bf16(E), _bf16(U)
        el, ul = _bf16(E - eh), _bf16(U - uh)
        p = d(eh) @ d(uh) + d(eh) @ d(ul) + d(el) @ d(uh)
    elif model == "tf32":
        p = d(_tf32(E)) @ d(_tf32(U))
    elif model == "bf16":
        p = d(_bf16(E)) @ d(_bf16(U))
    else:
        raise ValueError(model)
    return p.astype(np.float32)


def column_loop_f32(W, U, bits, group, block, model):
    """The column loop in float32 with the trailing products under `model`;
    W and U in processing order.  Returns the codes (processing order)."""
    W = np.array(W, dtype=np.float32)
    U = np.asarray(U, dtype=np.float32)
    rows, n = W.shape
    maxq = (1 << bits) - 1
    G = group if group > 0 else n
    codes = np.zeros((rows, n), dtype=np.int64)
    E = np.zeros((rows, n), dtype=np.float32)
    s = z = None
    for i1 in range(0, n, block):
        i2 = min(i1 + block, n)
        Wb = W[:, i1:i2].copy()
        for j in range(i2 - i1):
            col = i1 + j
            if col % G == 0:
                hi = min(col + G, n)
                cur = np.concatenate([Wb[:, j:], W[:, i2:hi]], axis=1) if hi > i2 else Wb[:, j:hi - i1]
                s, z = go.group_params_f32(cur, maxq)
            q, dq = go.quantize_values_f32(Wb[:, j], s, z, maxq)
            e = ((Wb[:, j] - dq) / U[col, col]).astype(np.float32)
            Wb[:, j + 1:] -= np.outer(e, U[col, col + 1:i2]).astype(np.float32)
            codes[:, col] = q
            E[:, col] = e
        if i2 < n:
            W[:, i2:] -= product(E[:, i1:i2], U[i1:i2, i2:], model)
    return codes


def agreement(spec_name, n=1024, rows=128, tokens_per_feature=None, models=("fp32", "3xtf32", "3xbf16", "tf32",
                                                                            "bf16")):
    """Share of codes equal to the fp64 oracle's, per model, on a scaled copy
    of a synthetic workload (same value structure, n columns, rows rows, the
    workload's tokens per feature unless given)."""
    import synth_inputs as si

    base = si.SPECS[spec_name]
    tpf = tokens_per_feature if tokens_per_feature is not None else base.n_tok / base.n
    spec = si.scaled(base, rows=rows, n=n, n_tok=max(int(round(tpf * n)), 16))
    W, X = si.make_layer(spec, "cpu")
    Wd, Xd = W.double().numpy(), X.double().numpy()
    ref = go.gptq_layer(Wd, X=Xd, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                        act_order=spec.act_order)
    Wp, U = ref["W"], ref["U"]
    out = {}
    for m in models:
        c = column_loop_f32(Wp, U, spec.bits, spec.group, spec.block, m)
        out[m] = float(np.mean(c == ref["codes"][:, ref["perm"]]))
    return spec, out
