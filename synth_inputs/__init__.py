"""Seeded synthetic layer inputs for the GPTQ configurations.

Holds no arithmetic of the method: only random weights and calibration
activations with the shapes, dtypes and value structure of the workloads
(weights ~ N(0, 0.02); activations N(0, 1) with outlier channels scaled up, or
half-normal with a fraction of zeros, or with log-normal per-channel scales).
The pages calibrate on real text and real model weights; none are available,
so these seeded tensors stand in for them.  Both the CUDA path and the oracle
consume the same tensors (the oracle gets a host copy).

Random streams: weights use torch.Generator seeded with ``seed``, activations
``seed + 1000``; a generator lives on the device the tensors are made on, so a
given seed gives the same tensors on every run of that device type.
"""
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class LayerSpec:
    name: str
    rows: int
    n: int
    n_tok: int
    w_dtype: str = "bf16"          # "bf16" or "f32"
    x_kind: str = "outliers"       # "outliers" | "halfnormal_zeros" | "lognormal_scales"
    outlier_frac: float = 0.01
    outlier_scale: float = 20.0
    zero_frac: float = 0.0
    bits: int = 4
    group: int = 128
    damp: float = 0.01
    block: int = 128
    act_order: bool = False
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def weights(self):
        return self.rows * self.n


# The five workload families (shapes, bit widths, groups, damping, order).
SPECS = {
    # single 256x256 fp32 layer, 2048 tokens with log-normal channel scales, per-row 4-bit
    "layer256": LayerSpec("layer256", 256, 256, 2048, w_dtype="f32", x_kind="lognormal_scales", bits=4, group=0,
                          seed=0),
    # Llama-7B attention projection, 128 x 2048 tokens, 1% outlier channels x20, 4-bit g128
    "attn4096": LayerSpec("attn4096", 4096, 4096, 262144, outlier_frac=0.01, outlier_scale=20.0, bits=4,
                          group=128, seed=2),
    # Llama-7B MLP pair, 3-bit g128 with act-order
    "mlp_up": LayerSpec("mlp_up", 11008, 4096, 262144, bits=3, group=128, act_order=True, seed=3),
    "mlp_down": LayerSpec("mlp_down", 4096, 11008, 262144, x_kind="halfnormal_zeros", zero_frac=0.3, bits=3,
                          group=128, act_order=True, seed=3),
    # OPT-175B-shaped stress layers, 65536 tokens, 0.5% outliers x50
    "fc1_g128_3b": LayerSpec("fc1_g128_3b", 49152, 12288, 65536, outlier_frac=0.005, outlier_scale=50.0, bits=3,
                             group=128, seed=5),
    "fc2_g64_2b": LayerSpec("fc2_g64_2b", 12288, 49152, 65536, outlier_frac=0.005, outlier_scale=50.0, bits=2,
                            group=64, seed=5),
}

# 7B-shaped layer set: per block q,k,v,o (4096x4096), gate,up (11008x4096),
# down (4096x11008); one X per input group (qkv, o, gate/up, down).
LAYERSET_BLOCK = [("q", 4096, 4096, "qkv"), ("k", 4096, 4096, "qkv"), ("v", 4096, 4096, "qkv"),
                  ("o", 4096, 4096, "o"), ("gate", 11008, 4096, "gateup"), ("up", 11008, 4096, "gateup"),
                  ("down", 4096, 11008, "down")]


def scaled(spec, rows=None, n=None, n_tok=None, **kw):
    """The same value structure at other sizes (for tests the oracle finishes)."""
    d = dict(spec.__dict__)
    d.update({k: v for k, v in (("rows", rows), ("n", n), ("n_tok", n_tok)) if v is not None})
    d.update(kw)
    return LayerSpec(**d)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_weights(spec, device="cpu"):
    g = _gen(device, spec.seed)
    W = torch.randn((spec.rows, spec.n), generator=g, device=device, dtype=torch.float32) * 0.02
    return W.to(torch.bfloat16) if spec.w_dtype == "bf16" else W


def make_activations(spec, device="cpu", chunk=16384):
    """X [n_tok, n] in bf16 (fp32 draws rounded to nearest-even bf16)."""
    g = _gen(device, spec.seed + 1000)
    n = spec.n
    chan_scale = torch.ones(n, dtype=torch.float32, device=device)
    if spec.x_kind == "outliers":
        k = int(round(spec.outlier_frac * n))
        idx = torch.randperm(n, generator=g, device=device)[:k]
        chan_scale[idx] = spec.outlier_scale
    elif spec.x_kind == "lognormal_scales":
        chan_scale = torch.exp(torch.randn(n, generator=g, device=device, dtype=torch.float32))
    X = torch.empty((spec.n_tok, n), dtype=torch.bfloat16, device=device)
    for t0 in range(0, spec.n_tok, chunk):
        t1 = min(spec.n_tok, t0 + chunk)
        x = torch.randn((t1 - t0, n), generator=g, device=device, dtype=torch.float32)
        if spec.x_kind == "halfnormal_zeros":
            x = x.abs()
            keep = torch.rand((t1 - t0, n), generator=g, device=device, dtype=torch.float32) >= spec.zero_frac
            x = x * keep
        else:
            x = x * chan_scale
        X[t0:t1] = x.to(torch.bfloat16)
    return X


def make_layer(spec, device="cpu"):
    return make_weights(spec, device), make_activations(spec, device)


def layerset_block(block, n_tok=131072, bits=4, group=128):
    """One block of the 7B-shaped layer set: the four calibration inputs (one
    per input group, 1% outlier channels x20) and the seven weight matrices.

    Returns (inputs, layers): inputs maps an input group to the LayerSpec of
    its activations (rows unused); layers lists (name, LayerSpec of the
    weights, input group).  Seeds: input group g of block b uses 40000 + 4b + g
    (its activations draw from that + 1000), layer i uses 50000 + 8b + i.
    """
    groups = ["qkv", "o", "gateup", "down"]
    widths = {"qkv": 4096, "o": 4096, "gateup": 4096, "down": 11008}
    inputs = {g: LayerSpec(f"layerset.b{block}.{g}", 0, widths[g], n_tok, bits=bits, group=group,
                           seed=40000 + 4 * block + gi)
              for gi, g in enumerate(groups)}
    layers = [(name, LayerSpec(f"layerset.b{block}.{name}", rows, n, n_tok, bits=bits, group=group,
                               seed=50000 + 8 * block + i), g)
              for i, (name, rows, n, g) in enumerate(LAYERSET_BLOCK)]
    return inputs, layers

