"""Gloo tests (CPU, world sizes 1 to 3) of the multi-rank host logic: token shards,
the global normaliser and max-over-ranks timing.  Per-rank compute is the
oracle here (no GPU); the claim tested is that shard results combined with the
global count equal the single-process result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunked_kl_loss_tma_b200.dist import global_valid_count, max_over_ranks, shard_range


def test_shards_partition_tokens():
    for n in (0, 1, 7, 4096, 4099):
        for world in (1, 2, 3, 8):
            got = [shard_range(n, world, r) for r in range(world)]
            covered = [i for a, b in got for i in range(a, b)]
            assert covered == list(range(n))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(0)  # same full problem on every rank
        N, d, V, K, T = 13, 4, 17, 3, 1.4
        H = rng.normal(size=(N, d))
        W = rng.normal(scale=0.5, size=(V, d))
        t = rng.normal(size=(N, V))
        idx = np.argsort(-t, axis=1)[:, :K].astype(np.int32)
        logit = np.take_along_axis(t, idx, 1)
        lse = np.log(np.exp(t / T).sum(1))
        mask = (rng.random(N) > 0.3).astype(np.uint8)
        a, b = shard_range(N, world, rank)
        n_all = global_valid_count(int(mask[a:b].sum()))
        out = oracle.kl_loss(H[a:b], W, T=T, mask=mask[a:b], topk_idx=idx[a:b],
                             topk_logit=logit[a:b], teacher_lse=lse[a:b], normalizer=n_all)
        loss = torch.tensor([out["loss"]], dtype=torch.float64)
        dW = torch.tensor(out["dW"])
        dist.all_reduce(loss)
        dist.all_reduce(dW)
        slowest = max_over_ranks(float(rank + 1))
        if rank == 0:
            ref = oracle.kl_loss(H, W, T=T, mask=mask, topk_idx=idx, topk_logit=logit,
                                 teacher_lse=lse)
            q.put((float(loss.item()), ref["loss"], float(np.max(np.abs(dW.numpy() - ref["dW"]))),
                   n_all, int(mask.sum()), slowest))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_rank_shards_with_global_normalizer_match_single_process(world):
    """world ranks (3: shards of 5, 4 and 4 of the 13 tokens)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    loss, ref, dw_err, n_all, n_ref, slowest = res
    assert n_all == n_ref
    assert loss == pytest.approx(ref, rel=1e-12)
    assert dw_err < 1e-12
    assert slowest == float(world)


def _reduce_worker(rank, world, port, q):
    from chunked_kl_loss_tma_b200.dist import dW_shard_rows, reduce_scatter_rows, sum_over_ranks

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        V, d = 11, 3  # V not a multiple of the world size: the last block is short
        parts = [torch.arange(V * d, dtype=torch.float32).reshape(V, d) * (r + 1)
                 for r in range(world)]
        total = sum(parts)
        t = parts[rank].clone()
        sum_over_ranks(t)
        shard = reduce_scatter_rows(parts[rank].clone())
        a, b = dW_shard_rows(V, world, rank)
        q.put((rank, torch.equal(t, total), torch.equal(shard, total[a:b]), (a, b)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2])
def test_sum_and_reduce_scatter_helpers(world):
    """sum_over_ranks and reduce_scatter_rows (the head-gradient reductions of
    the token data-parallel form) over gloo, against the plain sums; a group of
    one gloo rank leaves the tensor as it is."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reduce_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] and r[2] for r in res), res
    assert [r[3] for r in res] == ([(0, 11)] if world == 1 else [(0, 6), (6, 11)])
