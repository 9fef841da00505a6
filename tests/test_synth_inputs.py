"""The seeded synthetic inputs: shapes, dtypes, value structure and seeds of
the workloads (no arithmetic of the method lives there)."""
import torch

import synth_inputs as si


def test_specs_have_the_workload_shapes():
    s = si.SPECS
    assert (s["layer256"].rows, s["layer256"].n, s["layer256"].n_tok, s["layer256"].group) == (256, 256, 2048, 0)
    assert (s["attn4096"].rows, s["attn4096"].n, s["attn4096"].n_tok) == (4096, 4096, 262144)
    assert (s["attn4096"].bits, s["attn4096"].group, s["attn4096"].act_order) == (4, 128, False)
    assert (s["mlp_up"].rows, s["mlp_up"].n, s["mlp_up"].bits, s["mlp_up"].act_order) == (11008, 4096, 3, True)
    assert (s["mlp_down"].rows, s["mlp_down"].n, s["mlp_down"].x_kind) == (4096, 11008, "halfnormal_zeros")
    assert (s["fc1_g128_3b"].rows, s["fc1_g128_3b"].n, s["fc1_g128_3b"].n_tok) == (49152, 12288, 65536)
    assert (s["fc2_g64_2b"].bits, s["fc2_g64_2b"].group) == (2, 64)


def test_small_layer_is_seeded_and_structured():
    spec = si.scaled(si.SPECS["attn4096"], rows=32, n=200, n_tok=512)
    W, X = si.make_layer(spec, "cpu")
    W2, X2 = si.make_layer(spec, "cpu")
    assert W.dtype == torch.bfloat16 and X.dtype == torch.bfloat16
    assert W.shape == (32, 200) and X.shape == (512, 200)
    assert torch.equal(W, W2) and torch.equal(X, X2)
    # 1% of the channels (2 of 200) are scaled x20: their spread stands out
    std = X.float().std(dim=0)
    assert int((std > 5.0).sum()) == 2
    assert abs(W.float().std().item() - 0.02) < 0.004


def test_halfnormal_zeros_and_lognormal_kinds():
    spec = si.scaled(si.SPECS["mlp_down"], rows=4, n=64, n_tok=2048)
    X = si.make_activations(spec, "cpu").float()
    assert X.min().item() >= 0.0
    assert abs((X == 0).float().mean().item() - 0.3) < 0.03
    spec = si.scaled(si.SPECS["layer256"], rows=4, n=64, n_tok=1024)
    X = si.make_activations(spec, "cpu").float()
    std = X.std(dim=0)
    assert std.max().item() / std.min().item() > 3.0  # log-normal channel scales


def test_layerset_block_shapes_and_seeds():
    inputs, layers = si.layerset_block(3, n_tok=64)
    assert {g: s.n for g, s in inputs.items()} == {"qkv": 4096, "o": 4096, "gateup": 4096, "down": 11008}
    assert [s.seed for s in inputs.values()] == [40012, 40013, 40014, 40015]
    shapes = {name: (s.rows, s.n, g) for name, s, g in layers}
    assert shapes["q"] == (4096, 4096, "qkv") and shapes["gate"] == (11008, 4096, "gateup")
    assert shapes["down"] == (4096, 11008, "down")
    assert len({s.seed for _, s, _ in layers}) == 7
    assert sum(s.rows * s.n for _, s, _ in layers) * 32 == 6476005376
