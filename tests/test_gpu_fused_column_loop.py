"""The fused row-slab column loop (one launch per 1024-column super-block, a
CTA taking its rows through every block with left-looking corrections) against
the oracle's plain block loop.

GPTQ knowledge note, "How It Works": one column order for all rows, 128-column
blocks that accumulate their corrections before one global update; the fused
kernel applies the same corrections in another order (every column receives
every earlier column's correction before it is quantized), so the bar is the
layer tests' one: >= 99.9% of codes equal and the layer output error within
1e-3 of the oracle's.  The path is taken for n >= 2048 with 128-column blocks
whose groups divide 128 (or one group per row) and at most 32 rows per SM,
once gptq_set_column_loop(1) selects it.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si
from oracle import gptq_oracle as go

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq


@pytest.fixture(autouse=True)
def fused_loop():
    gq.gptq_set_column_loop(1)
    yield
    gq.gptq_set_column_loop(0)


def np64(t):
    return t.detach().double().cpu().numpy()


def _check(spec, rows_checked=None):
    W, X = si.make_layer(spec, "cuda")
    out = gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                            act_order=spec.act_order, want_deq=True, want_loss=True)
    torch.cuda.synchronize()
    Xh, Wh = np64(X), np64(W)
    idx = np.arange(spec.rows) if rows_checked is None else np.asarray(rows_checked)
    # the column loop treats every row on its own: the oracle on a subset of
    # rows gives those rows' codes
    ref = go.gptq_layer(Wh[idx], X=Xh, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                        act_order=spec.act_order)
    codes = out["codes"].cpu().numpy().astype(np.int64)[idx]
    agree = float(np.mean(codes == ref["codes"]))
    S = Xh.T @ Xh
    err_gpu = go.layer_output_error(Wh[idx], np64(out["deq"])[idx], S)
    err_ref = go.layer_output_error(Wh[idx], ref["deq"], S)
    return out, ref, agree, err_gpu, err_ref, idx


@pytest.mark.parametrize("name,rows,n,group", [
    ("attn4096", 48, 2048, 128),      # two full super-blocks
    ("attn4096", 33, 2176, 64),       # an odd row count; a last super-block of one block
    ("layer256", 30, 2100, 0),        # one group per row (its first block sees the rest); a 52-column last block
    ("fc2_g64_2b", 40, 2048, 64),     # 2-bit, groups of 64
    ("attn4096", 40, 2048, 32),       # groups of 32
    ("mlp_down", 36, 2304, 128),      # act-order, half-normal inputs with zero columns
])
def test_fused_column_loop_matches_oracle(name, rows, n, group):
    spec = si.scaled(si.SPECS[name], rows=rows, n=n, n_tok=4096, group=group, block=128)
    out, ref, agree, err_gpu, err_ref, _ = _check(spec)
    assert agree >= 0.999, agree
    assert abs(err_gpu - err_ref) <= 1e-3 * err_ref, (err_gpu, err_ref)
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=2e-2)
    if spec.act_order:
        assert np.array_equal(out["perm"].cpu().numpy().astype(np.int64), ref["perm"])


def test_fused_column_loop_full_slabs():
    """4,700 rows: 32-row slabs (the most one CTA takes), 147 CTAs; rows from
    the first, a middle and the last slab through the oracle."""
    spec = si.scaled(si.SPECS["attn4096"], rows=4700, n=2048, n_tok=4096, group=128, block=128)
    rows_checked = list(range(0, 8)) + list(range(2340, 2372)) + list(range(4690, 4700))
    out, ref, agree, err_gpu, err_ref, idx = _check(spec, rows_checked)
    assert agree >= 0.999, agree
    assert abs(err_gpu - err_ref) <= 1e-3 * err_ref, (err_gpu, err_ref)
