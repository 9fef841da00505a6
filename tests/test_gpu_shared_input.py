"""Layers that share one input (q/k/v, gate/up of the 7B-shaped layer set):
quantize_layer_group computes H and U once and quantizes every layer with
them; each layer must match the oracle's own run of that layer."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as go
import synth_inputs as si

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq


@pytest.mark.parametrize("act_order", [False, True])
def test_layer_group_matches_oracle_per_layer(act_order):
    base = si.scaled(si.SPECS["attn4096"], n=384, n_tok=4096, act_order=act_order)
    X = si.make_activations(base, "cuda")
    Ws = {name: si.make_weights(si.scaled(base, rows=rows, seed=50000 + i), "cuda")
          for i, (name, rows) in enumerate((("q", 48), ("k", 32), ("v", 64)))}
    out = gq.quantize_layer_group(Ws, X, bits=base.bits, group=base.group, damp=base.damp, block=base.block,
                                  act_order=act_order)
    torch.cuda.synchronize()
    Xh = X.double().cpu().numpy()
    S = Xh.T @ Xh
    for name, W in Ws.items():
        Wh = W.double().cpu().numpy()
        ref = go.gptq_layer(Wh, X=Xh, bits=base.bits, group=base.group, damp=base.damp, block=base.block,
                            act_order=act_order)
        res = out["layers"][name]
        codes = res["codes"].cpu().numpy().astype(np.int64)
        assert float(np.mean(codes == ref["codes"])) >= 0.999, name
        unpacked = go.unpack_codes(res["packed"].cpu().numpy().view(np.uint32), base.n, base.bits)
        assert np.array_equal(unpacked, codes), name
        G = base.group
        ng = -(-base.n // G)
        scales = res["scales"].cpu().numpy().astype(np.float64)
        zeros = res["zeros"].cpu().numpy().astype(np.float64)
        g_idx = res["g_idx"].cpu().numpy().astype(np.int64)
        assert scales.shape == (W.shape[0], ng)
        deq = scales[:, g_idx] * (codes - zeros[:, g_idx])
        err_gpu = go.layer_output_error(Wh, deq, S)
        err_ref = go.layer_output_error(Wh, ref["deq"], S)
        assert abs(err_gpu - err_ref) <= 1e-3 * err_ref, (name, err_gpu, err_ref)
    if act_order:
        assert np.array_equal(out["perm"].cpu().numpy().astype(np.int64), ref["perm"])
