"""One linear layer quantized by all ranks of a process group.

The pass shards along both of its natural axes (GPTQ knowledge note, "How It
Works": the Hessian H = 2 X X^T is a sum over calibration tokens, and every
output row follows the same column order with the same correction rows, so
rows are independent once U is known):

* tokens: each rank accumulates the Hessian of its own token shard with
  alpha = 2 / N, N the token count summed over the ranks; one all-reduce (sum)
  of H, and of the fp64 diagonal when act-order reads it, gives the layer's H
  on every rank;
* the factor: rank `root` runs gptq_prepare_hinv and broadcasts U, perm and
  dead, so that every rank quantizes with bit-identical factors (the
  factorization applies its trailing subtractions as L2 reductions, whose
  order of additions is not fixed, so two factorizations of one H may differ
  in the last bits);
* rows: each rank runs the column loop and the packing on its contiguous slice
  of rows, with no communication; ``gather=True`` assembles the full outputs
  on every rank with one all-gather per output.

Every rank must call ``quantize_layer_sharded`` with the same arguments except
its own slice of X (any number of tokens, possibly none).  The collectives are
torch.distributed's (NCCL for GPU tensors); all ranks issue them in the same
order.  W may be the full matrix or only this rank's rows (``w_is_local``).
"""
import torch
import torch.distributed as dist

from . import (LIB, gptq_hessian_accum, gptq_pack, gptq_prepare_hinv, gptq_quantize_layer, workspace)

__all__ = ["shard_range", "gather_rows", "quantize_layer_sharded"]


def shard_range(total, rank, world):
    """Contiguous slice [lo, hi) of `total` items owned by `rank` (sizes differ by at most one)."""
    return total * rank // world, total * (rank + 1) // world


def gather_rows(local, total, group=None):
    """All-gather of row slices: rank r contributes rows shard_range(total, r, world)
    of a [total, ...] tensor; every rank receives the whole tensor."""
    world = dist.get_world_size(group)
    per = -(-total // world)
    buf = torch.zeros((per,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    buf[: local.shape[0]] = local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    pieces = []
    for r in range(world):
        lo, hi = shard_range(total, r, world)
        pieces.append(parts[r][: hi - lo])
    return torch.cat(pieces, dim=0)


def quantize_layer_sharded(W, X_local, bits=4, group=128, damp=0.01, block=128, act_order=False,
                           process_group=None, root=0, w_is_local=False, gather=True):
    """Quantize one layer [rows, n] across the ranks of `process_group`.

    W        [rows, n] fp32/bf16 on this rank's GPU (or this rank's rows when
             w_is_local).
    X_local  [n_tok_r, n] bf16 on this rank's GPU: this rank's calibration tokens.
    Returns a dict with H, U, perm, dead, g_idx (identical on every rank), the
    row range ``rows`` = (lo, hi) of this rank, and codes, scales, zeros,
    packed, packed_zeros: the whole layer's when gather is True, else this
    rank's rows.
    """
    rank = dist.get_rank(process_group)
    world = dist.get_world_size(process_group)
    dev = X_local.device
    n = X_local.shape[1]

    # tokens: local Hessians with the global alpha, then one sum over the ranks
    count = torch.tensor([X_local.shape[0]], dtype=torch.float64, device=dev)
    dist.all_reduce(count, group=process_group)
    n_tok = int(count.item())
    if n_tok < 1:
        raise ValueError("no calibration tokens on any rank")
    H = torch.zeros((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.zeros(n, dtype=torch.float64, device=dev) if act_order else None
    if X_local.shape[0] > 0:
        gptq_hessian_accum(H, X_local, 2.0 / n_tok, hdiag=hdiag)
    dist.all_reduce(H, group=process_group)
    if hdiag is not None:
        dist.all_reduce(hdiag, group=process_group)

    # the factor: computed once, broadcast to every rank
    if rank == root:
        U, perm, dead = (t.contiguous() for t in gptq_prepare_hinv(H, damp, act_order, hdiag=hdiag))
    else:
        U = torch.empty((n, n), dtype=torch.float32, device=dev)
        perm = torch.empty(n, dtype=torch.int32, device=dev)
        dead = torch.empty(n, dtype=torch.uint8, device=dev)
    src = dist.get_global_rank(process_group, root) if process_group is not None else root
    for t in (U, perm, dead):
        dist.broadcast(t, src=src, group=process_group)

    # rows: this rank's slice through the column loop and the packing
    rows = W.shape[0] if not w_is_local else None
    if w_is_local:
        counts = torch.tensor([W.shape[0]], dtype=torch.float64, device=dev)
        dist.all_reduce(counts, group=process_group)
        rows = int(counts.item())
        lo, hi = shard_range(rows, rank, world)
        if W.shape[0] != hi - lo:
            raise ValueError(f"rank {rank} holds {W.shape[0]} rows, its slice is {hi - lo}")
        W_mine = W
    else:
        lo, hi = shard_range(rows, rank, world)
        W_mine = W[lo:hi]
    ng = LIB.gptq_num_groups(n, group)
    out = {"codes": torch.empty((hi - lo, n), dtype=torch.uint8, device=dev),
           "scales": torch.empty((hi - lo, ng), dtype=torch.float32, device=dev),
           "zeros": torch.empty((hi - lo, ng), dtype=torch.uint8, device=dev),
           "g_idx": torch.empty(n, dtype=torch.int32, device=dev)}
    if hi > lo:
        ws = workspace(LIB.gptq_quantize_workspace_size(hi - lo, n, block), dev)
        out = gptq_quantize_layer(W_mine, U, bits, group, block, perm=perm if act_order else None, dead=dead,
                                  out=out, ws=ws)
    out["packed"] = gptq_pack(out["codes"], bits) if hi > lo else torch.empty(
        (0, LIB.gptq_packed_words_per_row(n, bits)), dtype=torch.int32, device=dev)
    out["packed_zeros"] = gptq_pack(out["zeros"], bits) if hi > lo else torch.empty(
        (0, LIB.gptq_packed_words_per_row(ng, bits)), dtype=torch.int32, device=dev)
    # g_idx is written by the column loop; the last rank always has rows
    last = world - 1
    dist.broadcast(out["g_idx"], src=dist.get_global_rank(process_group, last) if process_group is not None
                   else last, group=process_group)
    if gather:
        for k in ("codes", "scales", "zeros", "packed", "packed_zeros"):
            out[k] = gather_rows(out[k], rows, process_group)
    out.update(H=H, U=U, perm=perm, dead=dead, rows=(lo, hi))
    return out
