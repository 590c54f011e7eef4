"""Token data-parallel form of the loss, and host-side helpers for multi-rank runs.

The loss partitions over tokens: each rank evaluates its own shard of rows
against the shared head with no collective on the data path.  Combining the
shards takes two exchanges.  The global count of valid tokens is summed first
and passed as `normalizer`, so every rank scales its loss and gradients by the
same mean.  Then the ranks' head gradients dW and their loss shares are summed
(all-reduce), or dW is reduce-scattered into row shards, as a sharded
optimizer keeps them.  dH stays with the rank that owns the tokens.

NCCL reduces device tensors in place, also in a group of one rank (so a one-GPU
run takes the multi-GPU path); another backend (gloo) stages them through host
memory, and a group of one gloo rank exchanges nothing."""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n_tokens: int, world: int, rank: int):
    """Contiguous, balanced [start, stop) token range of `rank` (sizes differ by
    at most one; together the ranges cover [0, n_tokens) exactly once)."""
    if world < 1 or not 0 <= rank < world or n_tokens < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_tokens, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _nccl(group):
    return dist.is_initialized() and dist.get_backend(group) == "nccl"


def global_valid_count(local_count: int, group=None) -> int:
    """Sum of the ranks' valid-token counts (one all-reduce of an int64)."""
    t = torch.tensor([int(local_count)], dtype=torch.int64)
    if _nccl(group):
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(t.item())


def max_over_ranks(value: float, group=None) -> float:
    """Max of a per-rank scalar (e.g. the elapsed time of the timed region)."""
    t = torch.tensor([float(value)], dtype=torch.float64)
    if _nccl(group):
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def dW_shard_rows(V: int, world: int, rank: int):
    """Rows [start, stop) of dW that `rank` holds after a reduce-scatter: V
    padded up to a multiple of `world`, equal blocks in rank order (the last
    block may hold fewer real rows)."""
    per = -(-V // world)
    start = min(rank * per, V)
    return start, min(start + per, V)


def sum_over_ranks(t: torch.Tensor, group=None, async_op: bool = False):
    """In-place sum of `t` over the ranks.  With NCCL and async_op, returns the
    work handle to wait on; otherwise the sum is complete on return."""
    if not dist.is_initialized() or (dist.get_world_size(group) == 1 and not _nccl(group)):
        return None
    if _nccl(group):
        return dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
    h = t.detach().to("cpu")
    dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
    t.copy_(h)
    return None


def reduce_scatter_rows(t: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of `t` [V, ...] over the ranks, returning this rank's block of rows
    (dW_shard_rows); a copy padded to the block size."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    if world == 1 and not _nccl(group):
        return t
    V = t.shape[0]
    per = -(-V // world)
    if per * world != V:
        pad = torch.zeros((per * world - V,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        t = torch.cat([t, pad])
    if _nccl(group):
        out = torch.empty((per,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.reduce_scatter_tensor(out, t.contiguous(), op=dist.ReduceOp.SUM, group=group)
        a, b = dW_shard_rows(V, world, rank)
        return out[: b - a]
    h = t.detach().to("cpu").contiguous()
    dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
    a, b = dW_shard_rows(V, world, rank)
    return h[a:b].to(t.device)


def dp_kl_fwd_bwd(H, W, *, group=None, grad_loss=1.0, mask=None, reduce="all_reduce",
                  dW=None, workspace=None, **kw):
    """Fused forward + backward of this rank's token shard H [n_r, d] against
    the shared head W, combined over the ranks of `group`.

    The normaliser is the global count of valid tokens (mask = 1 rows over all
    ranks), so the sum over ranks of the shard losses is the loss of the whole
    batch.  Returns dict(loss = the whole batch's loss, dH = this shard's rows,
    dW = the summed head gradient (reduce="all_reduce"), this rank's block of
    rows of it (reduce="reduce_scatter", rows dW_shard_rows(V, world, rank)) or
    the local gradient (reduce="none"), n_valid = the global count, workspace)."""
    from . import ops

    if reduce not in ("all_reduce", "reduce_scatter", "none"):
        raise ValueError(f"unknown reduce {reduce!r}")
    local = int(H.shape[0]) if mask is None else int(mask.sum().item())
    n_all = global_valid_count(local, group) if dist.is_initialized() else local
    out = ops.kl_fwd_bwd(H, W, grad_loss=grad_loss, mask=mask, normalizer=float(n_all), dW=dW,
                         workspace=workspace, **kw)
    loss = out["loss"].reshape(1)
    if reduce == "all_reduce":
        sum_over_ranks(out["dW"], group)
    elif reduce == "reduce_scatter":
        out["dW"] = reduce_scatter_rows(out["dW"], group)
    sum_over_ranks(loss, group)
    out["loss"] = loss.reshape(())
    out["n_valid"] = n_all
    return out
