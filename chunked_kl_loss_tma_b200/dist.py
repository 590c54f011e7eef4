"""Host-side helpers for running the loss data-parallel over tokens.

The loss partitions over tokens: each rank evaluates its own shard of rows
against the shared head with no collective on the data path.  Two small host
exchanges give a global result when one is wanted: the global count of valid
tokens (pass it as `normalizer` so every rank's loss and gradients are scaled
by the same mean), and the max over ranks of a measured time."""
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


def global_valid_count(local_count: int, group=None) -> int:
    """Sum of the ranks' valid-token counts (one all-reduce of an int64)."""
    t = torch.tensor([int(local_count)], dtype=torch.int64)
    if dist.is_initialized() and dist.get_backend(group) == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(t.item())


def max_over_ranks(value: float, group=None) -> float:
    """Max of a per-rank scalar (e.g. the elapsed time of the timed region)."""
    t = torch.tensor([float(value)], dtype=torch.float64)
    if dist.is_initialized() and dist.get_backend(group) == "nccl":
        t = t.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
