"""Expert parallelism over the GPUs of one node: expert e lives on GPU e mod G,
the router is replicated, and one exchange step surrounds the layer:

    x      [T, H] bf16 per GPU  --all-gather-->  [G*T, H] on every GPU
    moe_forward_partial on the gathered tokens (in chunks of at most one
        prefill chunk), remote experts contributing 0
    partial [G*T, H] fp32       --reduce-scatter (sum)-->  [T, H] per GPU
    moe_finish_rows: residual, steering, one bf16 rounding

The split applies to experts the multi-GPU layer split that the "Picking a
quant" page (multi-GPU section) gives as prior art.  This module is plumbing:
torch.distributed moves the tensors and every step of the layer's arithmetic
runs in libmoe.  The per-GPU sum is in slot order over the experts held there;
the cross-GPU sum is the collective's, so results match the single-GPU layer
within rounding, not bit for bit.
"""
from __future__ import annotations

from . import MOE_DECODE_MAX_T, MOE_PREFILL_MAX_T, MOE_SLOT_REMOTE, moe_finish_rows, moe_forward_partial


def ep_slot_table(slot_table, L: int, E: int, rank: int, G: int):
    """A copy of the [L][E] slot table (int32 tensor, any device) in which every
    expert not held by `rank` (e mod G != rank) is MOE_SLOT_REMOTE."""
    import torch
    t = slot_table.clone().view(L, E)
    remote = (torch.arange(E, device=t.device) % G) != rank
    t[:, remote] = MOE_SLOT_REMOTE
    return t.view(-1)


def _gather_rows(x, group):
    """[G*T, H] with rank r's rows at r*T .. r*T + T - 1.  The bf16 bits travel
    as int32 pairs (every backend moves 32-bit integers; H is even)."""
    import torch
    import torch.distributed as dist
    G = dist.get_world_size(group)
    x32 = x.contiguous().view(torch.int32)
    parts = [torch.empty_like(x32) for _ in range(G)]
    dist.all_gather(parts, x32, group=group)
    return torch.cat(parts, 0).view(x.dtype)


def _reduce_rows(partial, T: int, group):
    """Sum of every rank's partial [G*T, H]; this rank's rows [T, H]."""
    import torch
    import torch.distributed as dist
    rank = dist.get_rank(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((T,) + tuple(partial.shape[1:]), dtype=partial.dtype, device=partial.device)
        dist.reduce_scatter_tensor(out, partial, group=group)
        return out
    dist.all_reduce(partial, group=group)  # backends without reduce-scatter
    return partial[rank * T:(rank + 1) * T].contiguous()


def moe_forward_ep(desc, arena, slot_table_ep, L, layer, x, router_w, router_bias, top_k, residual, out,
                   group=None, prefill=None, steer=None, ws=None, hist=None, stream=None,
                   partial_fn=None, finish_fn=None, max_chunk=MOE_PREFILL_MAX_T):
    """One expert-parallel layer call on this rank's tokens x [T, H] (bf16 as
    int16), writing out [T, H].  slot_table_ep: this rank's table from
    ep_slot_table.  The G*T gathered tokens go through the library in chunks of
    at most max_chunk rows (one prefill chunk at most); prefill: the path for
    every chunk (default: the decode path for a chunk that fits it, else the
    chunk path).  ws must hold the workspace of one chunk.  partial_fn /
    finish_fn replace the two library calls (tests on CPU ranks) with
    partial_fn(x_chunk, partial_chunk) and finish_fn(x, total, out); by default
    they are moe_forward_partial and moe_finish_rows."""
    import torch
    import torch.distributed as dist
    if not 1 <= max_chunk <= MOE_PREFILL_MAX_T:
        raise ValueError(f"max_chunk must be in [1, {MOE_PREFILL_MAX_T}], got {max_chunk}")
    G = dist.get_world_size(group)
    T, H = x.shape
    x_all = _gather_rows(x, group)
    partial = torch.empty((G * T, H), dtype=torch.float32, device=x.device)
    for c0 in range(0, G * T, max_chunk):  # tokens are independent: any row split gives the same sums
        c1 = min(G * T, c0 + max_chunk)
        xc, pc = x_all[c0:c1], partial[c0:c1]
        if partial_fn is None:
            pf = (c1 - c0) > MOE_DECODE_MAX_T if prefill is None else prefill
            moe_forward_partial(pf, desc, arena, slot_table_ep, L, layer, xc, router_w, router_bias, top_k,
                                pc, hist=hist, ws=ws, stream=stream)
        else:
            partial_fn(xc, pc)
    total = _reduce_rows(partial, T, group)
    if finish_fn is None:
        moe_finish_rows(x, total, residual, out, steer=steer, stream=stream)
    else:
        finish_fn(x, total, out)
    return out
