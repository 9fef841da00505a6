"""Parity at full size for the other synthetic layers: the Llama-7B MLP pair
(3-bit g128 with act-order, 262,144 tokens) and the OPT-175B-shaped fc2
stress layer (12288 x 49152, 2-bit g64, 65,536 tokens with 0.5% outlier
channels x50), each through the public quantize_layer call.

Each check is one the oracle can afford at this size:
  * H on sampled entries, each an fp64 dot product of the same bf16 columns
    (relative Frobenius error over the sample <= 1e-3);
  * mlp_up: the oracle's whole fp64 pipeline (exact S over every token, its
    own damping, act-order and U) on sampled rows: >= 99.9% identical codes,
    the same permutation, the output error within 1e-3;
  * mlp_down: the oracle's factor and column loop on sampled rows from the
    GPU's H, with the act-order key the GPU used (its fp64 diagonal): the
    same permutation, >= 99.9% identical codes, output error within 1e-3;
  * fc2: U by probes (||U^T U H' v - v|| / ||v|| for random v, fp64 on the
    host), zeros below the diagonal; and the column loop on a column prefix:
    the first k codes of a row depend only on the leading k x k block of U
    (every correction reaching column j comes from columns i < j through
    U[i, j]), so the oracle runs its loop on W[:, :k] with the GPU's U[:k, :k]
    (>= 99.9% identical codes).
"""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as go
import synth_inputs as si

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_weight_quantization_accum_b200 as gq


def _h_sampled(X, H, n_tok, seed, count=2048):
    n = H.shape[0]
    rng = np.random.default_rng(seed)
    I = rng.integers(0, n, count)
    J = rng.integers(0, n, count)
    I[:64] = J[:64]
    Hg = H[torch.tensor(I, device="cuda"), torch.tensor(J, device="cuda")].double().cpu().numpy()
    ref = np.zeros(count)
    for a in range(0, count, 128):
        xi = X[:, torch.tensor(I[a:a + 128], device="cuda")].double().cpu().numpy()
        xj = X[:, torch.tensor(J[a:a + 128], device="cuda")].double().cpu().numpy()
        ref[a:a + 128] = np.float32(2.0 / n_tok) * np.einsum("ti,ti->i", xi, xj)
    return np.sqrt(np.sum((Hg - ref) ** 2) / np.sum(ref ** 2))


def _rows(out, W, rows):
    idx = torch.tensor(rows, device="cuda")
    return (W[idx].double().cpu().numpy(), out["codes"][idx].cpu().numpy().astype(np.int64),
            out["deq"][idx].double().cpu().numpy())


def test_mlp_up_full_pipeline_on_sampled_rows():
    spec = si.SPECS["mlp_up"]
    W, X = si.make_layer(spec, "cuda")
    out = gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                            act_order=spec.act_order, want_deq=True)
    torch.cuda.synchronize()
    assert _h_sampled(X, out["H"], spec.n_tok, 21) <= 1e-3
    n, N = spec.n, spec.n_tok
    S = np.zeros((n, n))
    for a in range(0, N, 16384):
        S = go.accumulate_hessian(S, X[a:a + 16384].double().cpu().numpy(), 1.0)
    rows = np.sort(np.random.default_rng(22).choice(spec.rows, 48, replace=False))
    Wh, codes, deq = _rows(out, W, rows)
    ref = go.gptq_layer(Wh, H=(2.0 / N) * S, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                        act_order=True)
    assert np.array_equal(out["perm"].cpu().numpy(), ref["perm"])
    assert float(np.mean(codes == ref["codes"])) >= 0.999
    e_gpu, e_ref = go.layer_output_error(Wh, deq, S), go.layer_output_error(Wh, ref["deq"], S)
    assert abs(e_gpu - e_ref) <= 1e-3 * e_ref, (e_gpu, e_ref)
    g_idx = out["g_idx"].cpu().numpy()
    assert np.array_equal(g_idx, ref["g_idx"])


def test_mlp_down_factor_and_loop_on_sampled_rows():
    spec = si.SPECS["mlp_down"]
    W, X = si.make_layer(spec, "cuda")
    n = spec.n
    # the public call, with the fp64 diagonal kept for the act-order key
    H = torch.zeros((n, n), device="cuda")
    hdiag = torch.zeros(n, dtype=torch.float64, device="cuda")
    gq.gptq_hessian_accum(H, X, 2.0 / spec.n_tok, hdiag=hdiag)
    U, perm, dead = gq.gptq_prepare_hinv(H, spec.damp, True, hdiag=hdiag)
    out = gq.gptq_quantize_layer(W, U, spec.bits, spec.group, spec.block, perm=perm, dead=dead, want_deq=True)
    torch.cuda.synchronize()
    assert gq.gptq_get_device_status() == 0
    assert _h_sampled(X, H, spec.n_tok, 31) <= 1e-3
    Hh = H.double().cpu().numpy()
    rows = np.sort(np.random.default_rng(32).choice(spec.rows, 48, replace=False))
    Wh, codes, deq = _rows(out, W, rows)
    ref = go.gptq_layer(Wh, H=Hh, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                        act_order=True, diag=hdiag.cpu().numpy())
    assert np.array_equal(perm.cpu().numpy(), ref["perm"])
    assert np.array_equal(dead.cpu().numpy().astype(bool), ref["dead"])
    assert float(np.mean(codes == ref["codes"])) >= 0.999
    S = Hh * (spec.n_tok / 2.0)
    e_gpu, e_ref = go.layer_output_error(Wh, deq, S), go.layer_output_error(Wh, ref["deq"], S)
    assert abs(e_gpu - e_ref) <= 1e-3 * e_ref, (e_gpu, e_ref)


def _matvec64(M, v, chunk=2048):
    """M (fp32, host) @ v in fp64, a row chunk at a time."""
    out = np.empty(M.shape[0])
    for a in range(0, M.shape[0], chunk):
        out[a:a + chunk] = M[a:a + chunk].astype(np.float64) @ v
    return out


def test_fc2_2bit_g64_probes_and_column_prefix():
    spec = si.SPECS["fc2_g64_2b"]
    W, X = si.make_layer(spec, "cuda")
    out = gq.quantize_layer(W, X, bits=spec.bits, group=spec.group, damp=spec.damp, block=spec.block,
                            act_order=False)
    torch.cuda.synchronize()
    n = spec.n
    assert _h_sampled(X, out["H"], spec.n_tok, 41) <= 1e-3
    del X
    Hh = out["H"].cpu().numpy()
    Uh = out["U"].cpu().numpy()
    # U by probes against the damped H (no act-order, no dead columns here)
    assert not out["dead"].any().item()
    lam = spec.damp * float(np.mean(np.diag(Hh).astype(np.float64)))
    rng = np.random.default_rng(42)
    for _ in range(2):
        v = rng.standard_normal(n)
        hv = _matvec64(Hh, v) + lam * v
        uhv = _matvec64(Uh, hv)
        r = _matvec64(np.ascontiguousarray(Uh.T), uhv) - v  # U^T (U (H' v)) - v
        assert np.linalg.norm(r) / np.linalg.norm(v) <= 1e-3
    tri = rng.integers(0, n, (4096, 2))
    lo = tri[tri[:, 0] > tri[:, 1]]
    assert np.all(Uh[lo[:, 0], lo[:, 1]] == 0.0)
    del Hh
    # the column loop on a prefix of k columns with the GPU's own U[:k, :k]
    k = 4096
    rows = np.sort(rng.choice(spec.rows, 32, replace=False))
    idx = torch.tensor(rows, device="cuda")
    Wp = W[idx, :k].double().cpu().numpy()
    ref = go.gptq_quantize(Wp, Uh[:k, :k].astype(np.float64), spec.bits, spec.group, spec.block)
    codes = out["codes"][idx, :k].cpu().numpy().astype(np.int64)
    assert float(np.mean(codes == ref["codes"])) >= 0.999
