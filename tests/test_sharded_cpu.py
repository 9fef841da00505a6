"""The sharded layer pass (post_weight_quantization_accum_b200.sharded) on CPU
gloo ranks: token shards summed by all-reduce, one factor broadcast, row shards
gathered.  The library calls are replaced, inside each spawned rank, by
stand-ins built from the fp64 oracle, so what is tested is the host logic:
the global alpha, the collectives, the shard ranges and the reassembly.  The
result must equal the oracle's run on the whole layer with the same Hessian.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed, rows, n, tokens):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((tokens, n)) * np.exp(rng.standard_normal(n))[None, :]).astype(np.float32)
    X[:, 3] = 0.0  # a dead column
    W = (0.02 * rng.standard_normal((rows, n))).astype(np.float32)
    return W, X


# --- stand-ins for the library calls (oracle arithmetic, CPU tensors) -------

def _hessian(H, X, alpha, hdiag=None, ws=None, stream=None):
    from oracle import gptq_oracle as go
    Xd = X.double().numpy()
    H += torch.from_numpy(go.hessian(Xd, alpha=alpha)).float()
    if hdiag is not None:
        hdiag += torch.from_numpy(alpha * np.sum(Xd * Xd, axis=0))
    return H


def _prepare(H, damp, act_order, hdiag=None, perm=None, dead=None, U=None, ws=None, stream=None):
    from oracle import gptq_oracle as go
    n = H.shape[0]
    diag = hdiag.numpy() if hdiag is not None else None
    prep = go.prepare(H.double().numpy(), np.zeros((1, n)), damp, act_order, diag=diag)
    Uf = torch.from_numpy(np.ascontiguousarray(go.inverse_factor(prep["H"]))).float()
    return Uf, torch.from_numpy(prep["perm"].astype(np.int32)), torch.from_numpy(prep["dead"].astype(np.uint8))


def _quantize(W, U, bits, group, block, perm=None, dead=None, out=None, want_deq=False, want_loss=False,
              ws=None, stream=None):
    from oracle import gptq_oracle as go
    n = W.shape[1]
    Wd = W.double().numpy().copy()
    Wd[:, dead.numpy().astype(bool)] = 0.0
    p = perm.numpy().astype(np.int64) if perm is not None else np.arange(n)
    res = go.gptq_quantize(Wd[:, p], U.double().numpy(), bits, group, block)
    codes = np.zeros(Wd.shape, dtype=np.int64)
    codes[:, p] = res["codes"]
    G = group if group > 0 else n
    g_idx = np.zeros(n, dtype=np.int64)
    g_idx[p] = np.arange(n) // G
    out["codes"].copy_(torch.from_numpy(codes.astype(np.uint8)))
    out["scales"].copy_(torch.from_numpy(res["scales"]).float())
    out["zeros"].copy_(torch.from_numpy(res["zeros"].astype(np.uint8)))
    out["g_idx"].copy_(torch.from_numpy(g_idx.astype(np.int32)))
    return out


def _pack(codes, bits, packed=None, stream=None):
    from oracle import gptq_oracle as go
    return torch.from_numpy(go.pack_codes(codes.numpy().astype(np.int64), bits).view(np.int32).copy())


def _worker(rank, world, port, q, case):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    import post_weight_quantization_accum_b200.sharded as sh
    sh.gptq_hessian_accum, sh.gptq_prepare_hinv = _hessian, _prepare
    sh.gptq_quantize_layer, sh.gptq_pack = _quantize, _pack
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        W, X = _inputs(case["seed"], case["rows"], case["n"], case["tokens"])
        t0, t1 = case["token_split"][rank], case["token_split"][rank + 1]
        Wt = torch.from_numpy(W)
        if case["w_is_local"]:
            lo, hi = sh.shard_range(case["rows"], rank, world)
            Wt = Wt[lo:hi].clone()
        out = sh.quantize_layer_sharded(Wt, torch.from_numpy(X[t0:t1]).to(torch.bfloat16), bits=case["bits"],
                                        group=case["group"], damp=0.01, block=case["block"],
                                        act_order=case["act_order"], root=case["root"],
                                        w_is_local=case["w_is_local"])
        q.put((rank, {k: out[k].numpy().copy() for k in ("codes", "scales", "zeros", "packed", "packed_zeros",
                                                          "g_idx", "perm", "U", "H")}, out["rows"]))
    finally:
        dist.destroy_process_group()


def _reference(case):
    """The whole layer through the same stand-ins, with H summed the way two
    fp32 partial Hessians are (the test's token splits give at most two
    non-empty shards, so the fp32 sum is order-independent)."""
    W, X = _inputs(case["seed"], case["rows"], case["n"], case["tokens"])
    Xb = torch.from_numpy(X).to(torch.bfloat16)
    n = case["n"]
    H = torch.zeros((n, n))
    hdiag = torch.zeros(n, dtype=torch.float64) if case["act_order"] else None
    parts = []
    for a, b in zip(case["token_split"][:-1], case["token_split"][1:]):
        Hp = torch.zeros((n, n))
        dp = torch.zeros(n, dtype=torch.float64) if case["act_order"] else None
        if b > a:
            _hessian(Hp, Xb[a:b], 2.0 / case["tokens"], hdiag=dp)
        parts.append((Hp, dp))
    for Hp, dp in parts:
        H += Hp
        if hdiag is not None:
            hdiag += dp
    U, perm, dead = _prepare(H, 0.01, case["act_order"], hdiag=hdiag)
    ng = -(-n // case["group"])
    out = {"codes": torch.empty((case["rows"], n), dtype=torch.uint8),
           "scales": torch.empty((case["rows"], ng)), "zeros": torch.empty((case["rows"], ng), dtype=torch.uint8),
           "g_idx": torch.empty(n, dtype=torch.int32)}
    _quantize(torch.from_numpy(W), U, case["bits"], case["group"], case["block"], perm=perm, dead=dead, out=out)
    return out, U, H


CASES = {
    "two ranks, act-order, uneven tokens": dict(seed=1, rows=24, n=96, tokens=400, token_split=[0, 150, 400],
                                               bits=3, group=32, block=32, act_order=True, root=0,
                                               w_is_local=False),
    "three ranks, a rank without rows or tokens, local rows, root 2": dict(
        seed=2, rows=2, n=64, tokens=300, token_split=[0, 0, 120, 300], bits=4, group=16, block=32,
        act_order=False, root=2, w_is_local=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_sharded_layer_equals_whole_layer(name):
    case = CASES[name]
    world = len(case["token_split"]) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, case)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, res, rows = q.get(timeout=180)
        got[rank] = (res, rows)
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    ref, U, H = _reference(case)
    from oracle import gptq_oracle as go
    for rank in range(world):
        res, rows = got[rank]
        assert rows == tuple(int(v) for v in (case["rows"] * rank // world, case["rows"] * (rank + 1) // world))
        assert np.array_equal(res["H"], H.numpy())
        assert np.array_equal(res["U"], U.numpy())           # every rank holds the root's factor
        assert np.array_equal(res["codes"], ref["codes"].numpy())
        assert np.array_equal(res["scales"], ref["scales"].numpy())
        assert np.array_equal(res["zeros"], ref["zeros"].numpy())
        assert np.array_equal(res["g_idx"], ref["g_idx"].numpy())
        packed = go.pack_codes(ref["codes"].numpy().astype(np.int64), case["bits"]).view(np.int32)
        assert np.array_equal(res["packed"], packed)
        assert np.array_equal(res["packed_zeros"],
                              go.pack_codes(ref["zeros"].numpy().astype(np.int64), case["bits"]).view(np.int32))


def test_shard_range_partitions():
    from post_weight_quantization_accum_b200.sharded import shard_range
    for total in (0, 1, 2, 7, 24, 4096):
        for world in (1, 2, 3, 8):
            spans = [shard_range(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
            assert spans[-1][1] - spans[-1][0] >= (1 if total >= 1 else 0)
