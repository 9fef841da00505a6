"""gptq_quantize_layer_noalloc: the column loop for callers that cannot allocate.

Some callers cannot give the library a workspace (they may not call cudaMalloc
or cudaFree, or all device memory belongs to a host application's pool).  The
allocation-free entry point keeps its scratch in a fixed device array inside
the library.  This test calls it through the C ABI twice in a row (the second
call finds the first call's leftovers in the shared array) and checks both
results against gptq_quantize_layer with a caller-provided workspace, within
the parity tests' bar for integer work: identical.  It also checks that a
layer too large for the fixed array is refused before any work.

The file name sorts last so that a run stopping at the first failure has run
every other test first.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq
    import synth_inputs as si

    _fn = gq.LIB.gptq_quantize_layer_noalloc
    _P = ctypes.c_void_p
    _fn.restype = ctypes.c_int
    _fn.argtypes = [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32, _P, _P, _P, ctypes.c_int32, ctypes.c_int32,
                    ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P]

SCRATCH_BYTES = 16 << 20


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _noalloc(W, U, perm, dead, bits, group, block):
    rows, n = W.shape
    ng = gq.LIB.gptq_num_groups(n, group)
    out = {"codes": torch.full((rows, n), 255, dtype=torch.uint8, device="cuda"),
           "scales": torch.full((rows, ng), float("nan"), device="cuda"),
           "zeros": torch.full((rows, ng), 255, dtype=torch.uint8, device="cuda"),
           "g_idx": torch.full((n,), -1, dtype=torch.int32, device="cuda"),
           "deq": torch.full((rows, n), float("nan"), device="cuda"),
           "row_loss": torch.full((rows,), float("nan"), device="cuda")}
    st = _fn(_p(W), gq.GPTQ_BF16 if W.dtype == torch.bfloat16 else gq.GPTQ_F32, rows, n, _p(U), _p(perm), _p(dead),
             bits, group, block, _p(out["codes"]), _p(out["scales"]), _p(out["zeros"]), _p(out["g_idx"]),
             _p(out["deq"]), _p(out["row_loss"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


@pytest.mark.parametrize("act_order", [False, True])
def test_noalloc_matches_workspace_entry_point_twice(act_order):
    spec = si.scaled(si.SPECS["mlp_up"], rows=384, n=1024, n_tok=4096, bits=3, group=128, act_order=act_order)
    W, X = si.make_layer(spec, "cuda")
    X[:, 5] = 0  # a dead column
    H = torch.zeros((spec.n, spec.n), device="cuda")
    hdiag = torch.zeros(spec.n, dtype=torch.float64, device="cuda")
    gq.gptq_hessian_accum(H, X, 2.0 / spec.n_tok, hdiag=hdiag)
    U, perm, dead = gq.gptq_prepare_hinv(H, spec.damp, act_order, hdiag=hdiag)
    p = perm if act_order else None
    ref = gq.gptq_quantize_layer(W, U, spec.bits, spec.group, spec.block, perm=p, dead=dead, want_deq=True,
                                 want_loss=True)
    for _ in range(2):
        st, out = _noalloc(W, U, p, dead, spec.bits, spec.group, spec.block)
        torch.cuda.synchronize()
        assert st == 0, st
        for k in ("codes", "zeros", "g_idx"):
            assert torch.equal(out[k], ref[k]), k
        for k in ("scales", "deq", "row_loss"):
            assert torch.equal(out[k], ref[k]), k


def test_noalloc_rejects_layers_beyond_its_scratch():
    rows, n = 2048, 2048   # needs 21 MiB of scratch
    assert gq.LIB.gptq_quantize_workspace_size(rows, n, 128) > SCRATCH_BYTES
    W = torch.zeros((rows, n), device="cuda")
    U = torch.eye(n, device="cuda")
    st, _ = _noalloc(W, U, None, None, 4, 128, 128)
    assert st == 1  # GPTQ_ERR_INVALID_ARG
    assert gq.LIB.gptq_quantize_workspace_size(1024, 1024, 128) <= SCRATCH_BYTES
