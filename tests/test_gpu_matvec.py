"""Inference with the packed weights (the next row after the quantization
pass): gptq_dequant_matvec against the oracle's fp64 dequant_matvec.

Tolerance: per run of 32 columns in one group the kernel forms
s * (sum_i code_i x_i - z * sum_i x_i) in fp32; each lane adds its runs
sequentially and the warp adds 32 lane sums in a 5-level tree.  The terms
being rounded are s * code * x and s * z * x (not their difference), so the
error is bounded by ~(32 k + 40) * eps * sum_c |s| (|code_c| + |z|) |x_c|
(k = runs per lane <= 16 here, eps = 2^-24); the bar uses 5e-5 times that sum
(a margin of ~5 over (32 * 16 + 40) * 6e-8 = 3.3e-5 in the worst case).
"""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as go

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq


def _case(rows, n, bits, group, batch, act_order, xdtype, seed, offset=0, zero_codes=False):
    """`offset` widens the bound's magnitude for kernels that round
    s * (offset + code) * x terms (the tensor-core path: offset 256 covers both
    its 128 + code and 128 + z terms)."""
    rng = np.random.default_rng(seed)
    maxq = (1 << bits) - 1
    G = group if group > 0 else n
    ng = -(-n // G)
    codes = rng.integers(0, maxq + 1, size=(rows, n))
    scales = rng.uniform(0.001, 0.02, size=(rows, ng)).astype(np.float32)
    zeros = rng.integers(0, maxq + 1, size=(rows, ng))
    if zero_codes:
        codes[:] = 0
        zeros[:] = 0
    g_idx = rng.permutation(np.arange(n) // G) if act_order else None
    x = rng.standard_normal((batch, n)).astype(np.float32)
    if xdtype == torch.bfloat16:
        x = torch.tensor(x).to(torch.bfloat16).float().numpy()
    packed = go.pack_codes(codes, bits)
    dev = "cuda"
    y = gq.gptq_dequant_matvec(torch.tensor(packed.view(np.int32), device=dev),
                               torch.tensor(scales, device=dev), torch.tensor(zeros.astype(np.uint8), device=dev),
                               n, bits, group, torch.tensor(x, device=dev).to(xdtype),
                               g_idx=None if g_idx is None else torch.tensor(g_idx.astype(np.int32), device=dev))
    torch.cuda.synchronize()
    ref = go.dequant_matvec(packed, scales, zeros, n, bits, group, x, g_idx)
    g = g_idx if g_idx is not None else np.arange(n) // G
    mag = np.abs(scales.astype(np.float64)[:, g]) * (offset + codes + zeros[:, g])  # |s| (offset + |code| + |z|)
    bound = (4e-6 if offset else 5e-5) * (np.abs(x.astype(np.float64)) @ mag.T)
    return y.double().cpu().numpy(), ref, bound


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("group", [0, 32, 128])
def test_matvec_matches_oracle(bits, group):
    y, ref, bound = _case(100, 512, bits, group, 1, False, torch.float32, bits * 10 + group)
    assert np.all(np.abs(y - ref) <= bound)


@pytest.mark.parametrize("batch", [2, 3, 8])
def test_matvec_batched_bf16_inputs(batch):
    y, ref, bound = _case(64, 1024, 4, 128, batch, False, torch.bfloat16, batch)
    assert y.shape == ref.shape
    assert np.all(np.abs(y - ref) <= bound)


@pytest.mark.parametrize("rows,n,group,batch", [
    (1, 128, 0, 1), (37, 512, 0, 1), (100, 512, 32, 1), (64, 1024, 64, 5), (48, 2048, 256, 2),
    (20, 512, 384, 3), (17, 4096, 0, 8), (33, 9216, 128, 1), (64, 11008, 128, 4), (16, 16384, 128, 8),
    (4096, 4096, 128, 1)])
def test_matvec_tensor_core_path(rows, n, group, batch):
    """4-bit codes and bf16 x with n % 128 == 0: groups of a multiple of 128
    columns (or one group per row) take the mma.sync path (16-row tiles,
    128-column blocks, 4 blocks per warp and round, so n = 9216, 11008 and
    16384 take several rounds), groups of 32 and 64 the general kernel.
    Error of the mma.sync path: per block the fp32 sum of s (128 + code) x
    over 8 chained MMAs (each adding 16 exact products), then the warp's
    blocks (n / 1024) and the 8 warps in sequence, minus the offsets
    sum_q s (128 + z) X_q (X_q from 8-value sums in 16- and T-lane trees):
    at most ~(8 + n / 1024 + 8 + 12) eps sum |s| (256 + code + z) |x|
    <= 2.7e-6 of that sum for n <= 16384; the bar is 4e-6."""
    y, ref, bound = _case(rows, n, 4, group, batch, False, torch.bfloat16, rows + n + batch, offset=256)
    assert y.shape == ref.shape
    assert np.all(np.abs(y - ref) <= bound)


def test_matvec_tensor_core_path_zero_codes():
    # every code and zero point 0: the 128 offsets cancel to rounding noise
    y, ref, bound = _case(40, 1024, 4, 128, 2, False, torch.bfloat16, 5, offset=256, zero_codes=True)
    assert np.all(ref == 0)
    assert np.all(np.abs(y - ref) <= bound)


def test_matvec_act_order_group_map():
    y, ref, bound = _case(80, 384, 3, 128, 2, True, torch.float32, 7)
    assert np.all(np.abs(y - ref) <= bound)


@pytest.mark.parametrize("n,group", [(1, 0), (33, 0), (1000, 200), (100, 20), (20000, 0)])
def test_matvec_ragged_and_long_rows(n, group):
    # runs cut by n, groups that split runs, and rows longer than one staging pass
    y, ref, bound = _case(37, n, 4, group, 1, False, torch.float32, n)
    assert np.all(np.abs(y - ref) <= bound)


def test_matvec_of_a_quantized_layer():
    """End to end: quantize a layer, pack, multiply; equals deq @ x."""
    import synth_inputs as si
    spec = si.scaled(si.SPECS["attn4096"], rows=128, n=512, n_tok=2048)
    W, X = si.make_layer(spec, "cuda")
    out = gq.quantize_layer(W, X, bits=4, group=128, want_deq=True)
    x = torch.randn((2, 512), device="cuda")
    y = gq.gptq_dequant_matvec(out["packed"], out["scales"], out["zeros"], 512, 4, 128, x)
    ref = x.double() @ out["deq"].double().T
    torch.cuda.synchronize()
    s = out["scales"].double().repeat_interleave(128, dim=1)
    z = out["zeros"].double().repeat_interleave(128, dim=1)
    mag = s.abs() * (out["codes"].double() + z)
    bound = 5e-5 * (x.double().abs() @ mag.T)
    assert torch.all((y.double() - ref).abs() <= bound)


def test_matvec_rejects_bad_arguments():
    p = torch.zeros((4, 4), dtype=torch.int32, device="cuda")
    s = torch.ones((4, 1), device="cuda")
    z = torch.zeros((4, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(gq.GptqError):
        gq.gptq_dequant_matvec(p, s, z, 32, 5, 0, torch.ones(32, device="cuda"))  # bits
    with pytest.raises(gq.GptqError):
        gq.gptq_dequant_matvec(p, s, z, 32, 4, 0, torch.ones((9, 32), device="cuda"))  # batch
