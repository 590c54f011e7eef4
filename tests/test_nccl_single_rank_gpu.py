"""The multi-GPU forms' NCCL branches on one GPU: a process group of one NCCL
rank.  NCCL still runs every collective (all-reduce, reduce-scatter,
all-gather into a tensor, the asynchronous dH all-reduce and its wait), on
device tensors and the caller's stream, so the code that a multi-GPU run takes
is exercised end to end; with one rank each collective is a copy.

Checks, in a spawned process (the group is created and destroyed there):
* the token data-parallel form (`dist.dp_kl_fwd_bwd`, all-reduce and
  reduce-scatter of dW) returns bit for bit what `kl_fwd_bwd` returns on the
  same batch, and matches the fp64 oracle (loss relative error <= 1e-3,
  gradients max-abs error <= 2e-2 max|oracle|);
* the vocabulary-parallel form (`vp_kl_fwd_bwd`, one shard holding the whole
  head) in the teacher-hidden mode with a reverse-KL weight, whose pass takes
  both statistics exchanges, matches `kl_fwd_bwd` within the same bounds."""
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


def _close(got, ref, rel):
    got = got.double().cpu().numpy() if torch.is_tensor(got) else np.asarray(got, np.float64)
    ref = ref.double().cpu().numpy() if torch.is_tensor(ref) else np.asarray(ref, np.float64)
    return float(np.max(np.abs(got - ref))) <= rel * float(np.max(np.abs(ref))) + 1e-6


def _worker(port, q):
    import torch.distributed as dist

    import oracle
    from chunked_kl_loss_tma_b200 import ops
    from chunked_kl_loss_tma_b200 import workloads as wl
    from chunked_kl_loss_tma_b200.dist import dp_kl_fwd_bwd
    from chunked_kl_loss_tma_b200.vocab_parallel import TorchComm, vp_kl_fwd_bwd

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    res = {}
    try:
        res["nccl_branch"] = TorchComm().nccl
        w = wl.make_topk("nccl_dp", N=301, d=200, V=5003, K=16, d_t=64, T=1.3,
                         dtype=torch.bfloat16, w_std=0.05, tw_std=0.1, seed=71)
        m = torch.ones(w.N, dtype=torch.uint8)
        m[::5] = 0
        w.mask = m
        w = w.to("cuda")
        kw = dict(T=w.T, topk_idx=w.topk_idx, topk_logit=w.topk_logit,
                  teacher_lse=w.teacher_lse, chunk_tokens=64)
        plain = ops.kl_fwd_bwd(w.H, w.W, grad_loss=0.8, mask=w.mask, **kw)
        ref = oracle.kl_loss(w.H, w.W, T=w.T, mask=w.mask, mode="topk", topk_idx=w.topk_idx,
                             topk_logit=w.topk_logit, teacher_lse=w.teacher_lse, grad_loss=0.8)
        for reduce in ("all_reduce", "reduce_scatter"):
            out = dp_kl_fwd_bwd(w.H, w.W, grad_loss=0.8, mask=w.mask, reduce=reduce, **kw)
            torch.cuda.synchronize()
            res[reduce] = dict(
                status=ops.status(out["workspace"]),
                n=out["n_valid"] == ref["n_valid"],
                same=bool(torch.equal(out["loss"], plain["loss"]) and
                          torch.equal(out["dH"], plain["dH"]) and
                          torch.equal(out["dW"], plain["dW"])),
                loss=abs(float(out["loss"]) - ref["loss"]) <= 1e-3 * abs(ref["loss"]),
                dH=_close(out["dH"], ref["dH"], 2e-2), dW=_close(out["dW"], ref["dW"], 2e-2))

        h = wl.make_hidden("nccl_vp", N=150, d=96, d_t=64, V=1700, T=1.7,
                           dtype=torch.bfloat16, w_std=0.08, tw_std=0.1, seed=72).to("cuda")
        hk = dict(T=h.T, Ht=h.Ht, reverse_weight=0.4, chunk_tokens=64)
        base = ops.kl_fwd_bwd(h.H, h.W, Wt=h.Wt, grad_loss=1.1, **hk)
        vp = vp_kl_fwd_bwd(h.H, h.W, v_begin=0, V_total=h.V, grad_loss=1.1, Wt=h.Wt, **hk)
        torch.cuda.synchronize()
        res["vp"] = dict(
            loss=abs(float(vp["loss"]) - float(base["loss"])) <= 1e-3 * abs(float(base["loss"])),
            dH=_close(vp["dH"], base["dH"], 2e-2), dW=_close(vp["dW"], base["dW"], 2e-2))
        q.put(res)
    except Exception as e:  # report instead of leaving the parent waiting
        q.put(dict(error=repr(e)))
    finally:
        dist.destroy_process_group()


def test_nccl_branches_in_a_one_rank_group():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=120)
    assert "error" not in res, res
    assert res["nccl_branch"]
    for reduce in ("all_reduce", "reduce_scatter"):
        r = res[reduce]
        assert r["status"] == 0 and r["n"], (reduce, r)
        assert r["same"], (reduce, "one-rank NCCL result differs from kl_fwd_bwd")
        assert r["loss"] and r["dH"] and r["dW"], (reduce, r)
    assert all(res["vp"].values()), res["vp"]
