"""B200 (sm_100a) GPTQ per-layer quantization: Python binding of libgptq_b200.so.

The functions below carry the names of the C entry points in include/gptq.h
and only marshal arguments: torch supplies device memory and the current CUDA
stream, the library's kernels do all of the work.  ``quantize_layer`` chains the
four calls for one linear layer (the usual entry point for a user);
``gptq2d_round`` is the two-sided rounding of the GPTQ-2D abstract.
"""
import ctypes

import torch

from ._lib import GPTQ_BF16, GPTQ_F32, LIB, GptqError, TraceEntry, check  # noqa: F401

__all__ = [
    "GptqError",
    "gptq_hessian_accum",
    "gptq_prepare_hinv",
    "gptq_quantize_layer",
    "gptq_quantize_rtn",
    "gptq_pack",
    "gptq_dequant_matvec",
    "gptq2d_round",
    "gptq2d_check_args",
    "gptq2d_factor",
    "gptq_get_device_status",
    "gptq_set_wait_limit_ns",
    "gptq_set_column_loop",
    "gptq_get_column_loop",
    "gptq_kernel_launches",
    "gptq_trace_enable",
    "gptq_trace_read",
    "workspace",
    "quantize_layer",
    "quantize_layer_group",
]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return GPTQ_F32
    if t.dtype == torch.bfloat16:
        return GPTQ_BF16
    raise TypeError(f"unsupported weight dtype {t.dtype}")


def workspace(nbytes, device=None):
    """A 256-byte aligned device buffer of at least ``nbytes`` (torch memory)."""
    return torch.empty(max(int(nbytes), 1) + 256, dtype=torch.uint8, device=device or "cuda")


def _ws_ptr(ws):
    base = ws.data_ptr()
    return ctypes.c_void_p((base + 255) & ~255), ws.numel() - ((-base) % 256)


def gptq_get_device_status(stream=None):
    return LIB.gptq_get_device_status(_stream(stream))


def gptq_set_wait_limit_ns(ns):
    LIB.gptq_set_wait_limit_ns(ctypes.c_uint64(ns))


def gptq_set_column_loop(mode):
    """0: per-block kernels (default); 1: the fused row-slab pass where it applies."""
    LIB.gptq_set_column_loop(int(mode))


def gptq_get_column_loop():
    return int(LIB.gptq_get_column_loop())


def gptq_kernel_launches():
    return int(LIB.gptq_kernel_launches())


def gptq_trace_enable(on=True):
    LIB.gptq_trace_enable(1 if on else 0)


def gptq_trace_read(max_entries=64):
    """{kernel name: (launches, device ms)} since the previous read (waits for
    the traced launches to finish)."""
    buf = (TraceEntry * max_entries)()
    n = LIB.gptq_trace_read(buf, max_entries)
    if n < 0:
        raise GptqError("gptq_trace_read", 4)
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].ms)) for i in range(n)}


def gptq_hessian_accum(H, X, alpha, hdiag=None, ws=None, stream=None):
    """H += alpha * X^T X (X bf16 [n_tok, n] view with unit column stride); hdiag fp64 optional."""
    if X.dtype != torch.bfloat16 or X.stride(1) != 1:
        raise TypeError("X must be a bf16 matrix with contiguous rows")
    n_tok, ldx = X.shape[0], X.stride(0)
    n = H.shape[0]
    need = LIB.gptq_hessian_workspace_size(n, n_tok)
    if ws is None:
        ws = workspace(need, H.device)
    wp, wbytes = _ws_ptr(ws)
    check("gptq_hessian_accum",
          LIB.gptq_hessian_accum(_ptr(H), _ptr(hdiag), _ptr(X), n_tok, n, ldx, ctypes.c_float(alpha), wp,
                                 wbytes, _stream(stream)))
    return H


def gptq_prepare_hinv(H, damp, act_order, hdiag=None, perm=None, dead=None, U=None, ws=None, stream=None):
    """Returns (U, perm, dead) for the accumulated Hessian H (fp32 [n, n])."""
    n = H.shape[0]
    dev = H.device
    U = U if U is not None else torch.empty((n, n), dtype=torch.float32, device=dev)
    perm = perm if perm is not None else torch.empty(n, dtype=torch.int32, device=dev)
    dead = dead if dead is not None else torch.empty(n, dtype=torch.uint8, device=dev)
    if ws is None:
        ws = workspace(LIB.gptq_prepare_workspace_size(n), dev)
    wp, wbytes = _ws_ptr(ws)
    check("gptq_prepare_hinv",
          LIB.gptq_prepare_hinv(_ptr(H), _ptr(hdiag), n, ctypes.c_float(damp), int(bool(act_order)), _ptr(perm),
                                _ptr(dead), _ptr(U), wp, wbytes, _stream(stream)))
    return U, perm, dead


def gptq_quantize_layer(W, U, bits, group, block=128, perm=None, dead=None, out=None, want_deq=False,
                        want_loss=False, ws=None, stream=None):
    """The GPTQ column loop; returns a dict of output tensors."""
    rows, n = W.shape
    dev = W.device
    ng = LIB.gptq_num_groups(n, group)
    out = dict(out or {})
    out.setdefault("codes", torch.empty((rows, n), dtype=torch.uint8, device=dev))
    out.setdefault("scales", torch.empty((rows, ng), dtype=torch.float32, device=dev))
    out.setdefault("zeros", torch.empty((rows, ng), dtype=torch.uint8, device=dev))
    out.setdefault("g_idx", torch.empty(n, dtype=torch.int32, device=dev))
    if want_deq:
        out.setdefault("deq", torch.empty((rows, n), dtype=torch.float32, device=dev))
    if want_loss:
        out.setdefault("row_loss", torch.empty(rows, dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(LIB.gptq_quantize_workspace_size(rows, n, block), dev)
    wp, wbytes = _ws_ptr(ws)
    check("gptq_quantize_layer",
          LIB.gptq_quantize_layer(_ptr(W), _dtype_code(W), rows, n, _ptr(U), _ptr(perm), _ptr(dead), bits, group,
                                  block, _ptr(out["codes"]), _ptr(out["scales"]), _ptr(out["zeros"]),
                                  _ptr(out.get("g_idx")), _ptr(out.get("deq")), _ptr(out.get("row_loss")), wp,
                                  wbytes, _stream(stream)))
    return out


def gptq_quantize_rtn(W, bits, group, stream=None):
    rows, n = W.shape
    dev = W.device
    ng = LIB.gptq_num_groups(n, group)
    codes = torch.empty((rows, n), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, ng), dtype=torch.float32, device=dev)
    zeros = torch.empty((rows, ng), dtype=torch.uint8, device=dev)
    check("gptq_quantize_rtn",
          LIB.gptq_quantize_rtn(_ptr(W), _dtype_code(W), rows, n, bits, group, _ptr(codes), _ptr(scales),
                                _ptr(zeros), _stream(stream)))
    return {"codes": codes, "scales": scales, "zeros": zeros}


def gptq_pack(codes, bits, packed=None, stream=None):
    rows, n = codes.shape
    words = LIB.gptq_packed_words_per_row(n, bits)
    if packed is None:
        packed = torch.empty((rows, words), dtype=torch.int32, device=codes.device)
    check("gptq_pack", LIB.gptq_pack(_ptr(codes), rows, n, bits, _ptr(packed), _stream(stream)))
    return packed


def gptq_dequant_matvec(packed, scales, zeros, n, bits, group, x, g_idx=None, y=None, ws=None, stream=None):
    """y[b, r] = sum_c Q[r, c] x[b, c] with Q read from the packed rows; x is
    [batch, n] (or [n]) fp32 or bf16 on the device; returns fp32 [batch, rows]."""
    rows = packed.shape[0]
    squeeze = x.dim() == 1
    x2 = x.reshape(1, -1) if squeeze else x
    batch = x2.shape[0]
    xdt = _dtype_code(x2)
    if y is None:
        y = torch.empty((batch, rows), dtype=torch.float32, device=packed.device)
    need = LIB.gptq_matvec_workspace_size(n, batch, xdt)
    wp, wb = ctypes.c_void_p(0), 0
    if need > 0:
        wp, wb = _ws_ptr(ws if ws is not None else workspace(need, packed.device))
    x2 = x2.contiguous()
    check("gptq_dequant_matvec", LIB.gptq_dequant_matvec(_ptr(packed), _ptr(scales), _ptr(zeros), _ptr(g_idx), rows,
                                                         n, bits, group, _ptr(x2), xdt, batch, _ptr(y), wp, wb,
                                                         _stream(stream)))
    return y[0] if squeeze else y


def gptq2d_factor(H, damp=0.0, ws=None, stream=None):
    """Upper U with U^T U = (H + damp * mean(diag H) I)^-1 for a symmetric
    positive definite Gram H (fp32 [k, k]): gptq_prepare_hinv without
    reordering (damp 0: the Gram as given)."""
    U, _, _ = gptq_prepare_hinv(H, damp, False, ws=ws, stream=stream)
    return U


def gptq2d_check_args(W, UL, UR, qmin=None, qmax=None):
    """The checks gptq2d_round makes before it touches the device (shapes,
    dtypes, row-major layout); they need no GPU, so callers can run them on
    host tensors built the same way."""
    m, n = W.shape
    if (qmin is None) != (qmax is None):
        raise ValueError("give both qmin and qmax, or neither")
    if tuple(UL.shape) != (m, m) or tuple(UR.shape) != (n, n):
        raise ValueError(f"factors {tuple(UL.shape)} and {tuple(UR.shape)} do not match W {tuple(W.shape)}")
    if W.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"unsupported weight dtype {W.dtype}")
    if UL.dtype != torch.float32 or UR.dtype != torch.float32:
        raise TypeError("UL and UR must be fp32")
    if not (W.is_contiguous() and UL.is_contiguous() and UR.is_contiguous()):
        raise ValueError("W, UL and UR must be contiguous row-major matrices")


def gptq2d_round(W, UL, UR, scale=1.0, qmin=None, qmax=None, want_E=True, codes=None, E=None, ws=None,
                 stream=None):
    """Two-sided GPTQ (GPTQ-2D): round W [m, n] (fp32 or bf16) to scale * integers
    under tr(HL D HR D^T), given the upper factors UL (UL^T UL = HL^-1) and UR
    (UR^T UR = HR^-1).  Clamps the integers to [qmin, qmax] when both are given.
    Returns dict(codes=int32 [m, n], E=fp32 [m, n] scaled errors or None)."""
    gptq2d_check_args(W, UL, UR, qmin, qmax)
    m, n = W.shape
    dev = W.device
    clamp = 0 if qmin is None else 1
    codes = codes if codes is not None else torch.empty((m, n), dtype=torch.int32, device=dev)
    if want_E and E is None:
        E = torch.empty((m, n), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(LIB.gptq2d_workspace_size(m, n), dev)
    wp, wbytes = _ws_ptr(ws)
    check("gptq2d_round",
          LIB.gptq2d_round(_ptr(W), _dtype_code(W), m, n, _ptr(UL), _ptr(UR), ctypes.c_float(scale), clamp,
                           int(qmin or 0), int(qmax or 0), _ptr(codes), _ptr(E), wp, wbytes, _stream(stream)))
    return {"codes": codes, "E": E}


def _hessian_from_host(H, X, hdiag, stream, chunk_tokens):
    """H += (2/N) X^T X for calibration inputs in host memory: token chunks are
    copied into two device buffers on a copy stream while the library
    accumulates the previous chunk, so the transfer and the SYRK overlap.
    (Pinned host memory makes the copies asynchronous.)"""
    n_tok, n = X.shape
    dev = H.device
    compute = stream if stream is not None else torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    pitch = (n + 7) // 8 * 8
    m = min(chunk_tokens, n_tok)
    bufs = [torch.empty((m, pitch), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    ws = workspace(LIB.gptq_hessian_workspace_size(n, m), dev)
    ws.record_stream(compute)
    alpha = 2.0 / n_tok
    for i, t0 in enumerate(range(0, n_tok, m)):
        k = i % 2
        rows = min(m, n_tok - t0)
        if i >= 2:
            copy.wait_event(free[k])
        with torch.cuda.stream(copy):
            bufs[k][:rows, :n].copy_(X[t0:t0 + rows], non_blocking=True)
            ready[k].record(copy)
        compute.wait_event(ready[k])
        gptq_hessian_accum(H, bufs[k][:rows, :n], alpha, hdiag=hdiag, ws=ws, stream=compute)
        free[k].record(compute)
        bufs[k].record_stream(compute)
    return H


def _raise_on_device_status(stream):
    # A bounded in-kernel wait that ran out leaves the asynchronous calls'
    # status at GPTQ_OK but records GPTQ_ERR_TIMEOUT on the device; read (and
    # clear) it so that such a run cannot hand back wrong codes silently.
    code = gptq_get_device_status(stream)
    if code != 0:
        raise GptqError("device status", code)


def quantize_layer(W, X, bits=4, group=128, damp=0.01, block=128, act_order=False, want_deq=False,
                   want_loss=False, stream=None, device=None, chunk_tokens=16384, check=True):
    """One linear layer end to end: H from X, U, the column loop, packing.

    W: [rows, n] fp32/bf16 weights; X: [n_tok, n] bf16 calibration inputs.
    Either may live in host memory (ideally pinned): X is then streamed to the
    GPU in chunks of `chunk_tokens` tokens, each chunk's SYRK overlapping the
    copy of the next.  Everything is computed on `device` (default: W's device
    if W is on a GPU, else the current one).  Returns a dict of device tensors
    with H, U, perm, codes, scales, zeros, g_idx, packed, packed_zeros (and deq
    / row_loss when asked for).  With ``check`` (the default) the call ends by
    reading the library's device status word, which synchronizes the stream,
    and raises GptqError if a bounded in-kernel wait ran out.
    """
    n = W.shape[1]
    dev = torch.device(device) if device is not None else (W.device if W.is_cuda else
                                                             torch.device("cuda", torch.cuda.current_device()))
    if not W.is_cuda:
        W = W.to(dev, non_blocking=True)
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if act_order else None
    if not X.is_cuda:
        _hessian_from_host(H, X, hdiag, stream, chunk_tokens)
    else:
        if X.stride(1) != 1 or X.stride(0) % 8 != 0 or X.data_ptr() % 16 != 0:
            # the library streams X with TMA, whose row pitch must be a multiple
            # of 16 bytes: hand it a row-padded copy
            Xp = torch.zeros((X.shape[0], (n + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)
            Xp[:, :n] = X
            X = Xp[:, :n]
        gptq_hessian_accum(H, X, 2.0 / X.shape[0], hdiag=hdiag, stream=stream)
    U, perm, dead = gptq_prepare_hinv(H, damp, act_order, hdiag=hdiag, stream=stream)
    out = gptq_quantize_layer(W, U, bits, group, block, perm=perm if act_order else None, dead=dead,
                              want_deq=want_deq, want_loss=want_loss, stream=stream)
    out["packed"] = gptq_pack(out["codes"], bits, stream=stream)
    out["packed_zeros"] = gptq_pack(out["zeros"], bits, stream=stream)
    out.update(H=H, U=U, perm=perm, dead=dead)
    if check:
        _raise_on_device_status(stream)
    return out


def quantize_layer_group(Ws, X, bits=4, group=128, damp=0.01, block=128, act_order=False, stream=None,
                         device=None, chunk_tokens=16384, check=True):
    """Several layers that read the same input (e.g. the q, k and v projections):
    H, the damping, act-order and U depend only on X, so they are computed once
    and every layer's column loop and packing reuse them.

    Ws: dict name -> W [rows_i, n]; X: [n_tok, n] bf16 (device or host).
    Returns dict(H, U, perm, dead, layers={name: outputs as in quantize_layer});
    ``check`` as in quantize_layer.
    """
    first = next(iter(Ws.values()))
    n = first.shape[1]
    if any(W.shape[1] != n for W in Ws.values()):
        raise ValueError("every layer of a group must have X's width as its column count")
    dev = torch.device(device) if device is not None else (first.device if first.is_cuda else
                                                             torch.device("cuda", torch.cuda.current_device()))
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if act_order else None
    if not X.is_cuda:
        _hessian_from_host(H, X, hdiag, stream, chunk_tokens)
    else:
        if X.stride(1) != 1 or X.stride(0) % 8 != 0 or X.data_ptr() % 16 != 0:
            Xp = torch.zeros((X.shape[0], (n + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)
            Xp[:, :n] = X
            X = Xp[:, :n]
        gptq_hessian_accum(H, X, 2.0 / X.shape[0], hdiag=hdiag, stream=stream)
    U, perm, dead = gptq_prepare_hinv(H, damp, act_order, hdiag=hdiag, stream=stream)
    layers = {}
    for name, W in Ws.items():
        if not W.is_cuda:
            W = W.to(dev, non_blocking=True)
        out = gptq_quantize_layer(W, U, bits, group, block, perm=perm if act_order else None, dead=dead,
                                  stream=stream)
        out["packed"] = gptq_pack(out["codes"], bits, stream=stream)
        out["packed_zeros"] = gptq_pack(out["zeros"], bits, stream=stream)
        layers[name] = out
    if check:
        _raise_on_device_status(stream)
    return {"H": H, "U": U, "perm": perm, "dead": dead, "layers": layers}

