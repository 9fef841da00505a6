"""quantize_layer_group's host logic on the CPU: the Hessian, the damping and
the factor are computed once per shared input and every layer's column loop
reads them.  The library calls are replaced by counting stand-ins (the
oracle's arithmetic), so no GPU is involved."""
import numpy as np
import torch

import post_weight_quantization_accum_b200 as gq
from oracle import gptq_oracle as go


def test_group_computes_h_and_u_once_and_quantizes_every_layer(monkeypatch):
    calls = {"h": 0, "p": 0, "q": [], "pack": 0, "status": 0}
    rng = np.random.default_rng(3)
    n, n_tok = 48, 300
    X = torch.from_numpy(rng.standard_normal((n_tok, n)).astype(np.float32)).to(torch.bfloat16)
    Ws = {name: torch.from_numpy((0.02 * rng.standard_normal((rows, n))).astype(np.float32))
          for name, rows in (("q", 16), ("k", 8), ("v", 24))}

    def hessian_from_host(H, Xh, hdiag, stream, chunk_tokens):
        calls["h"] += 1
        H += torch.from_numpy(go.hessian(Xh.double().numpy())).float()
        return H

    def prepare(H, damp, act_order, hdiag=None, perm=None, dead=None, U=None, ws=None, stream=None):
        calls["p"] += 1
        prep = go.prepare(H.double().numpy(), np.zeros((1, n)), damp, act_order)
        U = torch.from_numpy(np.ascontiguousarray(go.inverse_factor(prep["H"]))).float()
        return U, torch.from_numpy(prep["perm"].astype(np.int32)), torch.from_numpy(prep["dead"].astype(np.uint8))

    def quantize(W, U, bits, group, block, perm=None, dead=None, out=None, stream=None, **kw):
        calls["q"].append(U)
        res = go.gptq_quantize(W.double().numpy(), U.double().numpy(), bits, group, block)
        return {"codes": torch.from_numpy(res["codes"].astype(np.uint8)),
                "zeros": torch.from_numpy(res["zeros"].astype(np.uint8)),
                "scales": torch.from_numpy(res["scales"]).float()}

    def pack(codes, bits, packed=None, stream=None):
        calls["pack"] += 1
        return torch.from_numpy(go.pack_codes(codes.numpy().astype(np.int64), bits).view(np.int32).copy())

    monkeypatch.setattr(gq, "_hessian_from_host", hessian_from_host)
    monkeypatch.setattr(gq, "gptq_prepare_hinv", prepare)
    monkeypatch.setattr(gq, "gptq_quantize_layer", quantize)
    monkeypatch.setattr(gq, "gptq_pack", pack)

    def status(stream=None):
        calls["status"] += 1
        return 0

    monkeypatch.setattr(gq, "gptq_get_device_status", status)
    out = gq.quantize_layer_group(Ws, X, bits=3, group=16, damp=0.01, block=16, device="cpu")
    assert calls["h"] == 1 and calls["p"] == 1 and calls["pack"] == 2 * len(Ws)
    assert calls["status"] == 1  # the device status word is read once, at the end
    assert len(calls["q"]) == len(Ws) and all(U is out["U"] for U in calls["q"])
    for name, W in Ws.items():
        ref = go.gptq_layer(W.double().numpy(), X=X.double().numpy(), bits=3, group=16, damp=0.01, block=16)
        assert np.array_equal(out["layers"][name]["codes"].numpy(), ref["codes"])
        assert np.array_equal(out["layers"][name]["packed"].numpy(),
                              go.pack_codes(ref["codes"], 3).view(np.int32))
