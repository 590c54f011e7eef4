"""Token data-parallel form with the CUDA path: two or three processes share one GPU and
exchange over gloo (host-side collectives, so neither rank's kernels wait on
the other's).  Each rank runs its token shard through kl_fwd_bwd with the
global count of valid tokens as the normaliser; the head gradient and the loss
shares are then summed (or dW reduce-scattered into row blocks).  The result
must be the whole batch's: loss, every rank's dH rows and dW against the fp64
oracle on the unsharded problem, with the tolerances of the other parity tests
(loss relative error <= 1e-3, gradients max-abs error <= 2e-2 max|oracle|)."""
import os
import socket

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, reduce, q):
    import torch.distributed as dist

    import oracle
    from chunked_kl_loss_tma_b200 import ops
    from chunked_kl_loss_tma_b200 import workloads as wl
    from chunked_kl_loss_tma_b200.dist import dp_kl_fwd_bwd, dW_shard_rows, shard_range

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        # the same batch on every rank (same seed); each rank keeps its rows
        w = wl.make_topk("dp", N=301, d=200, V=5003, K=16, d_t=64, T=1.3,
                         dtype=torch.bfloat16, w_std=0.05, tw_std=0.1, seed=61)
        m = torch.ones(w.N, dtype=torch.uint8)
        m[::5] = 0
        w.mask = m
        w = w.to("cuda")
        a, b = shard_range(w.N, world, rank)
        out = dp_kl_fwd_bwd(w.H[a:b], w.W, grad_loss=0.8, mask=w.mask[a:b], reduce=reduce,
                            T=w.T, topk_idx=w.topk_idx[a:b], topk_logit=w.topk_logit[a:b],
                            teacher_lse=w.teacher_lse[a:b], chunk_tokens=64)
        torch.cuda.synchronize()
        ref = oracle.kl_loss(w.H, w.W, T=w.T, mask=w.mask, mode="topk", topk_idx=w.topk_idx,
                             topk_logit=w.topk_logit, teacher_lse=w.teacher_lse, grad_loss=0.8)
        v0, v1 = (0, w.V) if reduce == "all_reduce" else dW_shard_rows(w.V, world, rank)
        dW = out["dW"].double().cpu().numpy()
        q.put(dict(rank=rank, status=ops.status(out["workspace"]), n=out["n_valid"],
                   n_ref=ref["n_valid"], loss=float(out["loss"]), ref_loss=ref["loss"],
                   dH=float(np.max(np.abs(out["dH"].double().cpu().numpy() - ref["dH"][a:b]))),
                   dH_scale=float(np.max(np.abs(ref["dH"]))),
                   dW_rows=dW.shape[0], dW_rows_ref=v1 - v0,
                   dW=float(np.max(np.abs(dW - ref["dW"][v0:v1]))),
                   dW_scale=float(np.max(np.abs(ref["dW"])))))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put(dict(rank=rank, error=repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("reduce,world", [("all_reduce", 2), ("reduce_scatter", 2),
                                          ("reduce_scatter", 3)])
def test_token_shards_over_gloo_on_one_gpu(reduce, world):
    """world processes (3: uneven token shards, and dW row blocks of a V that 3
    does not divide)."""
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, reduce, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in res:
        assert "error" not in r, r
        assert r["status"] == 0 and r["n"] == r["n_ref"], r
        assert abs(r["loss"] - r["ref_loss"]) <= 1e-3 * abs(r["ref_loss"]), r
        assert r["dH"] <= 2e-2 * r["dH_scale"], r
        assert r["dW_rows"] == r["dW_rows_ref"], r
        assert r["dW"] <= 2e-2 * r["dW_scale"], r
