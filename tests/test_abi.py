"""The C-ABI library loads on the CPU and exports every entry point its header
declares; pure (non-compute) calls answer without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")
LIB = os.path.join(ROOT, "post_weight_quantization_accum_b200", "libgptq_b200.so")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq\w*)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()  # compiles only if a source is newer than the library
    return ctypes.CDLL(LIB)


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("gptq_hessian_accum", "gptq_prepare_hinv", "gptq_quantize_layer", "gptq_pack", "gptq_dequant_matvec",
              "gptq2d_round", "gptq2d_workspace_size"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_pure_calls(lib):
    lib.gptq_packed_words_per_row.restype = ctypes.c_int32
    assert lib.gptq_packed_words_per_row(4096, 4) == 512
    assert lib.gptq_packed_words_per_row(33, 3) == 6
    assert lib.gptq_packed_words_per_row(10, 5) == 0
    assert lib.gptq_num_groups(4096, 128) == 32
    assert lib.gptq_num_groups(100, 0) == 1
    assert lib.gptq_num_groups(129, 64) == 3
    lib.gptq_status_string.restype = ctypes.c_char_p
    assert lib.gptq_status_string(2) == b"damped Hessian is not positive definite"
    assert lib.gptq_version() == 100


def test_column_loop_selector(lib):
    """gptq_set_column_loop: 0 (per-block loop) by default, 1 selects the fused
    row-slab pass, anything else falls back to 0; the setting needs no GPU."""
    lib.gptq_get_column_loop.restype = ctypes.c_int32
    lib.gptq_set_column_loop.argtypes = [ctypes.c_int32]
    assert lib.gptq_get_column_loop() == 0
    try:
        lib.gptq_set_column_loop(1)
        assert lib.gptq_get_column_loop() == 1
        for other in (2, -1, 7):
            lib.gptq_set_column_loop(other)
            assert lib.gptq_get_column_loop() == 0
    finally:
        lib.gptq_set_column_loop(0)


def test_invalid_arguments_rejected_before_any_launch(lib):
    P = ctypes.c_void_p
    f = lib.gptq_quantize_layer
    f.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32, P, P, P, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    fake = P(256)
    # bits 5, block 48, group/block not nesting, bad dtype
    assert f(fake, 0, 8, 64, fake, None, None, 5, 0, 128, fake, fake, fake, None, None, None, fake, 1 << 30, None) == 1
    assert f(fake, 0, 8, 64, fake, None, None, 4, 0, 48, fake, fake, fake, None, None, None, fake, 1 << 30, None) == 1
    assert f(fake, 0, 8, 96, fake, None, None, 4, 48, 64, fake, fake, fake, None, None, None, fake, 1 << 30, None) == 5
    assert f(fake, 7, 8, 64, fake, None, None, 4, 0, 64, fake, fake, fake, None, None, None, fake, 1 << 30, None) == 1
    g = lib.gptq_pack
    g.argtypes = [P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, P, P]
    assert g(None, 4, 64, 4, fake, None) == 1
    assert g(fake, 4, 64, 6, fake, None) == 1
    h = lib.gptq_hessian_accum
    h.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, P, ctypes.c_size_t, P]
    assert h(fake, None, fake, 128, 64, 60, 1.0, fake, 1 << 30, None) == 1    # ldx < n
    assert h(fake, None, fake, 128, 64, 68, 1.0, fake, 1 << 30, None) == 1    # ldx % 8
    assert h(fake, None, P(258), 128, 64, 64, 1.0, fake, 1 << 30, None) == 1  # X alignment
    assert h(fake, None, fake, 0, 64, 64, 1.0, None, 0, None) == 0            # no tokens: no-op
    p = lib.gptq_prepare_hinv
    p.argtypes = [P, P, ctypes.c_int32, ctypes.c_float, ctypes.c_int32, P, P, P, P, ctypes.c_size_t, P]
    assert p(fake, None, 64, -0.1, 0, None, None, fake, fake, 1 << 30, None) == 1
    assert p(fake, None, 64, 0.01, 1, None, None, fake, fake, 1 << 30, None) == 1  # act-order needs perm


def test_gptq2d_arguments_rejected_before_any_launch(lib):
    P = ctypes.c_void_p
    ws = lib.gptq2d_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [ctypes.c_int64, ctypes.c_int64]
    assert ws(64, 64) == 5 * 64 * 64 * 4   # W copy, the far and near push buffers, E
    assert ws(3, 5) == 5 * 256
    assert ws(-1, 5) == 0
    f = lib.gptq2d_round
    f.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, P, P, ctypes.c_float, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, P, P, P, ctypes.c_size_t, P]
    fake = P(256)
    big = 1 << 30
    assert f(fake, 0, -1, 8, fake, fake, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1   # negative size
    assert f(fake, 0, 8, 8, fake, fake, 0.0, 0, 0, 0, fake, None, fake, big, None) == 1    # scale 0
    assert f(fake, 0, 8, 8, fake, fake, float("nan"), 0, 0, 0, fake, None, fake, big, None) == 1
    assert f(fake, 0, 8, 8, fake, fake, 1.0, 2, 0, 0, fake, None, fake, big, None) == 1     # clamp flag
    assert f(fake, 0, 8, 8, fake, fake, 1.0, 1, 3, -3, fake, None, fake, big, None) == 1    # qmin > qmax
    assert f(fake, 0, 8, 8, fake, fake, 1.0, 1, -(1 << 25), 0, fake, None, fake, big, None) == 1
    assert f(fake, 3, 8, 8, fake, fake, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1     # dtype
    assert f(None, 0, 8, 8, fake, fake, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1     # W NULL
    assert f(fake, 0, 8, 8, fake, None, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1     # UR NULL
    assert f(P(258), 0, 8, 8, fake, fake, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1   # fp32 W alignment
    assert f(fake, 0, 8, 8, fake, fake, 1.0, 0, 0, 0, fake, None, fake, 100, None) == 1     # small workspace
    assert f(fake, 0, 8, 8, fake, fake, 1.0, 0, 0, 0, fake, None, P(384 + 64), big, None) == 1  # ws alignment
    assert f(fake, 0, 0, 8, fake, fake, 1.0, 0, 0, 0, fake, None, None, 0, None) == 0       # empty: no-op
    assert f(fake, 0, (1 << 22) + 1, 1, fake, fake, 1.0, 0, 0, 0, fake, None, fake, big, None) == 1


def test_binding_fails_loudly_without_the_library(tmp_path):
    from post_weight_quantization_accum_b200 import _lib
    with pytest.raises(ImportError, match="no fallback"):
        _lib.load(str(tmp_path / "libgptq_b200.so"))



def test_gptq2d_binding_checks_shapes_before_the_library():
    import torch
    import post_weight_quantization_accum_b200 as gq
    W = torch.zeros((3, 5))
    with pytest.raises(ValueError):
        gq.gptq2d_round(W, torch.eye(3), torch.eye(4))
    with pytest.raises(TypeError):
        gq.gptq2d_round(W, torch.eye(3, dtype=torch.float64), torch.eye(5))
    with pytest.raises(ValueError):
        gq.gptq2d_round(W, torch.eye(3), torch.eye(6)[:5, :5])   # a non-contiguous view
    with pytest.raises(ValueError):
        gq.gptq2d_round(W, torch.eye(3), torch.eye(5), qmin=-1)


def test_smoke_gptq2d_inputs_pass_the_binding_checks():
    """smoke() builds its GPTQ-2D inputs with the oracle's factor and
    torch.tensor; the same construction on the host must satisfy every check
    gptq2d_round makes before it touches the device (a non-contiguous factor
    once failed smoke on the GPU)."""
    import __graft_entry__ as ge
    import post_weight_quantization_accum_b200 as gq
    W2, UL, UR = ge.gptq2d_smoke_inputs()
    W, ULt, URt = ge.gptq2d_smoke_tensors(W2, UL, UR, "cpu")
    assert ULt.is_contiguous() and URt.is_contiguous()
    gq.gptq2d_check_args(W, ULt, URt)
