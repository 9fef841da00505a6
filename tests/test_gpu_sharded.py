"""The sharded layer pass (sharded.quantize_layer_sharded) on the real
library: two spawned ranks on the one GPU, a gloo process group over CUDA
tensors (no NCCL, no NVLS or multicast; the ranks' kernels never wait on one
another: every exchange is a host-side gloo collective).  Each rank holds half
of the calibration tokens; the token-sharded H, the broadcast factor and the
row-sharded column loop must reproduce the oracle's whole-layer run: the same
permutation and group indices, >= 99.9% identical codes, and the gathered
packed rows equal to packing the gathered codes."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir, act_order):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import synth_inputs as si
    from post_weight_quantization_accum_b200 import sharded

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    spec = si.scaled(si.SPECS["mlp_up"], rows=300, n=640, n_tok=6000, act_order=act_order)
    W, X = si.make_layer(spec, "cuda")
    lo, hi = sharded.shard_range(spec.n_tok, rank, world)
    out = sharded.quantize_layer_sharded(W, X[lo:hi].contiguous(), bits=spec.bits, group=spec.group,
                                         damp=spec.damp, block=spec.block, act_order=act_order)
    torch.cuda.synchronize()
    if rank == 0:
        torch.save({k: (v.cpu() if torch.is_tensor(v) else v) for k, v in out.items()},
                   os.path.join(outdir, "out.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("act_order", [False, True])
def test_two_ranks_on_one_gpu_match_the_oracle(act_order):
    import synth_inputs as si
    from oracle import gptq_oracle as go

    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_main, args=(2, _free_port(), d, act_order), nprocs=2, join=True)
        out = torch.load(os.path.join(d, "out.pt"))
    spec = si.scaled(si.SPECS["mlp_up"], rows=300, n=640, n_tok=6000, act_order=act_order)
    W, X = si.make_layer(spec, "cuda")  # the ranks' inputs (the generators are device-specific)
    W, X = W.cpu(), X.cpu()
    ref = go.gptq_layer(W.double().numpy(), X=X.double().numpy(), bits=spec.bits, group=spec.group,
                        damp=spec.damp, block=spec.block, act_order=act_order)
    codes = out["codes"].numpy().astype(np.int64)
    assert codes.shape == (spec.rows, spec.n)
    assert np.array_equal(out["perm"].numpy(), ref["perm"])
    assert np.array_equal(out["g_idx"].numpy(), ref["g_idx"])
    assert float(np.mean(codes == ref["codes"])) >= 0.999
    assert np.array_equal(out["packed"].numpy().view(np.uint32), go.pack_codes(codes, spec.bits))
