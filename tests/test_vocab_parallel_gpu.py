"""Vocabulary-parallel form (head split by rows over P ranks), emulated on one
GPU: the P shards run one after another, each through kl_vp_fwd_chunk /
kl_vp_bwd_chunk with its own workspace, the exchange of row statistics is a
concatenation and the sums over ranks are additions.  The merged result must
match the fp64 oracle of the whole problem (same tolerances as the whole-head
tests), and a single shard covering the whole head must reproduce kl_fwd_bwd
bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import vocab_parallel as vp
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
GRAD_FRAC = 2e-2


def _topk(N=300, d=200, V=5003, K=16, dtype=torch.bfloat16, T=1.3, seed=31, partial=True):
    w = wl.make_topk("vp_topk", N=N, d=d, V=V, K=K, d_t=64, T=T, dtype=dtype, w_std=0.05,
                     tw_std=0.1, seed=seed, partial_mass=partial)
    m = torch.ones(N, dtype=torch.uint8)
    m[::7] = 0
    w.mask = m
    return w.to("cuda")


def _hidden(N=200, d=136, d_t=72, V=3001, dtype=torch.bfloat16, T=2.0, seed=32):
    w = wl.make_hidden("vp_hidden", N=N, d=d, d_t=d_t, V=V, T=T, dtype=dtype, w_std=0.08,
                       tw_std=0.1, seed=seed)
    m = torch.ones(N, dtype=torch.uint8)
    m[3::5] = 0
    w.mask = m
    return w.to("cuda")


def _kw(w, chunk=0):
    kw = dict(T=w.T, mask=w.mask, chunk_tokens=chunk)
    if w.mode == "topk":
        kw.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        kw.update(Ht=w.Ht, Wt=w.Wt)
    return kw


def _oracle(w, **kw):
    args = dict(T=w.T, mask=w.mask, mode=w.mode)
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    args.update(kw)
    return oracle.kl_loss(w.H, w.W, **args)


def _check_grad(got, ref, name):
    got = got.detach().double().cpu().numpy()
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(got - ref))
    assert err <= GRAD_FRAC * scale, f"{name}: max abs err {err:.3e} > {GRAD_FRAC} * {scale:.3e}"


def _check_all(out, ref):
    assert abs(float(out["loss"]) - ref["loss"]) <= LOSS_RTOL * abs(ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=5e-3,
                               atol=2e-4)
    np.testing.assert_allclose(out["lse_s"].cpu().numpy(), ref["lse_s"], rtol=1e-5, atol=1e-5)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    for ws in out["workspaces"]:
        assert ops.status(ws) == 0


# shard layouts over V = 5003: balanced on 256-row blocks, and ragged ones with
# a 3-row shard and boundaries inside tiles
TOPK_SHARDS = {
    "P2": None,
    "P3_ragged": [(0, 256), (256, 259), (259, 5003)],
    "P4_unaligned": [(0, 1000), (1000, 2500), (2500, 2501), (2501, 5003)],
}


@pytest.mark.parametrize("partial", [True, False])
@pytest.mark.parametrize("layout", list(TOPK_SHARDS))
def test_topk_shards_match_oracle(partial, layout):
    w = _topk(partial=partial)
    shards = TOPK_SHARDS[layout]
    P = 2 if shards is None else len(shards)
    out = vp.emulate(w.H, w.W, P, shards=shards, grad_loss=1.7, want_row_loss=True,
                     want_lse=True, **_kw(w, chunk=128))
    _check_all(out, _oracle(w, grad_loss=1.7))


@pytest.mark.parametrize("layout", ["P2", "P3_ragged"])
def test_topk_shards_fused_dlogits(layout):
    """Shards with dS formed inside each shard's dH contraction (fuse_dlogits),
    including a 3-row shard and boundaries inside tiles."""
    w = _topk(seed=37)
    shards = TOPK_SHARDS[layout]
    P = 2 if shards is None else len(shards)
    out = vp.emulate(w.H, w.W, P, shards=shards, grad_loss=1.1, want_row_loss=True,
                     want_lse=True, fuse_dlogits=True, **_kw(w, chunk=128))
    _check_all(out, _oracle(w, grad_loss=1.1))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_hidden_shards_match_oracle(dtype):
    w = _hidden(dtype=dtype)
    kw = _kw(w, chunk=96)
    Wt = kw.pop("Wt")
    out = vp.emulate(w.H, w.W, 3, shards=[(0, 1024), (1024, 1030), (1030, 3001)], Wt=Wt,
                     want_row_loss=True, want_lse=True, **kw)
    _check_all(out, _oracle(w))


@pytest.mark.parametrize("beta", [0.35, 1.0])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_reverse_kl_mixing_shards_match_oracle(beta, dtype):
    """Reverse-KL weight > 0: the second exchange (every shard's sums A, U)
    gives u_bar over the whole vocabulary before dS is written."""
    w = _hidden(dtype=dtype, seed=34)
    kw = dict(_kw(w, chunk=96), reverse_weight=beta)
    Wt = kw.pop("Wt")
    out = vp.emulate(w.H, w.W, 3, shards=[(0, 1024), (1024, 1030), (1030, 3001)], Wt=Wt,
                     grad_loss=1.3, want_row_loss=True, want_lse=True, **kw)
    _check_all(out, _oracle(w, reverse_weight=beta, grad_loss=1.3))


def test_reverse_kl_single_shard_is_the_fused_call_bit_for_bit():
    w = _hidden(seed=36)
    kw = dict(_kw(w, chunk=128), reverse_weight=0.5)
    ref = ops.kl_fwd_bwd(w.H, w.W, grad_loss=0.7, want_row_loss=True, **kw)
    Wt = kw.pop("Wt")
    out = vp.emulate(w.H, w.W, 1, Wt=Wt, grad_loss=0.7, want_row_loss=True, **kw)
    for k in ("loss", "row_loss", "dH", "dW"):
        assert torch.equal(out[k], ref[k]), k


def test_per_token_temperature_shards():
    g = torch.Generator().manual_seed(5)
    Tr = (0.5 + 2.5 * torch.rand(300, generator=g)).to(torch.float32)
    w = wl.make_topk("vp_ptt", N=300, d=200, V=5003, K=16, d_t=64, T=Tr, dtype=torch.bfloat16,
                     w_std=0.05, tw_std=0.1, seed=33).to("cuda")
    w.mask = torch.ones(300, dtype=torch.uint8, device="cuda")
    w.mask[::6] = 0
    out = vp.emulate(w.H, w.W, 2, want_row_loss=True, want_lse=True, **_kw(w, chunk=128))
    _check_all(out, _oracle(w))


@pytest.mark.parametrize("mode", ["topk", "hidden"])
def test_single_shard_is_the_fused_call_bit_for_bit(mode):
    w = _topk() if mode == "topk" else _hidden()
    kw = _kw(w, chunk=128)
    ref = ops.kl_fwd_bwd(w.H, w.W, grad_loss=0.7, want_row_loss=True, **kw)
    Wt = kw.pop("Wt", None)
    out = vp.emulate(w.H, w.W, 1, Wt=Wt, grad_loss=0.7, want_row_loss=True, **kw)
    assert torch.equal(out["loss"], ref["loss"])
    assert torch.equal(out["row_loss"], ref["row_loss"])
    assert torch.equal(out["dH"], ref["dH"])
    assert torch.equal(out["dW"], ref["dW"])


def test_cache_entries_outside_every_shard_of_a_row():
    # rows whose cached ids all fall in one shard: the other shards see none
    w = _topk(seed=35, K=8)
    idx = w.topk_idx.clone()
    idx[:50] = torch.arange(8, dtype=torch.int32, device="cuda")[None, :] + 4000
    idx[50:60, 4:] = -1                       # empty slots
    w.topk_idx = idx
    out = vp.emulate(w.H, w.W, 2, want_row_loss=True, want_lse=True, **_kw(w, chunk=0))
    _check_all(out, _oracle(w))


def test_out_of_range_cache_id_sets_status():
    w = _topk(seed=36)
    idx = w.topk_idx.clone()
    idx[5, 3] = w.V                           # outside the whole vocabulary
    w.topk_idx = idx
    out = vp.emulate(w.H, w.W, 2, **_kw(w))
    assert all(ops.status(ws) == 7 for ws in out["workspaces"])   # KL_ERR_INDEX


def test_accumulate_dW_and_empty_problem():
    w = _topk(seed=37)
    shards = vp.vocab_shard(w.V, 2, 0), vp.vocab_shard(w.V, 2, 1)
    base = torch.randn(w.W.shape, generator=torch.Generator().manual_seed(1)).cuda()
    full = vp.emulate(w.H, w.W, 2, **_kw(w, chunk=128))
    for r, (v0, v1) in enumerate(shards):
        s = vp.ShardPass(w.H, w.W[v0:v1], v_begin=v0, V_total=w.V, dW=base[v0:v1].clone(),
                         accumulate_dW=True, **_kw(w, chunk=128))
        # drive the shard with the other shard's statistics from a fresh pass
        other = vp.ShardPass(w.H, w.W[shards[1 - r][0]:shards[1 - r][1]],
                             v_begin=shards[1 - r][0], V_total=w.V, **_kw(w, chunk=128))
        for k in range(len(s.chunks)):
            mine, theirs = s.fwd_chunk(k), other.fwd_chunk(k)
            st = torch.cat([mine, theirs] if r == 0 else [theirs, mine])
            s.bwd_chunk(k, st, 2, r)
        torch.testing.assert_close(s.dW, base[v0:v1] + full["dW"][v0:v1], rtol=0, atol=1e-5)
    H0 = w.H[:0]
    out = vp.emulate(H0, w.W, 2, topk_idx=w.topk_idx[:0], topk_logit=w.topk_logit[:0],
                     teacher_lse=w.teacher_lse[:0], T=w.T)
    assert float(out["loss"]) == 0.0 and out["dH"].shape == (0, w.d)
    assert torch.count_nonzero(out["dW"]) == 0


def _free_port():
    import socket

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _two_rank_worker(rank, world, port, q):
    import os

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    # host-side gloo collectives: both ranks' kernels share one GPU and never
    # wait on each other inside a kernel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        w = _topk(seed=39)
        v0, v1 = vp.vocab_shard(w.V, world, rank)
        out = vp.vp_kl_fwd_bwd(w.H, w.W[v0:v1], v_begin=v0, V_total=w.V, grad_loss=1.2,
                               want_row_loss=True, want_lse=True, **_kw(w, chunk=128))
        torch.cuda.synchronize()
        ref = _oracle(w, grad_loss=1.2)
        dW = out["dW"].double().cpu().numpy()
        res = dict(rank=rank, status=ops.status(out["workspace"]),
                   loss=float(out["loss"]), ref_loss=ref["loss"],
                   # row losses: |got - ref| / (5e-3 |ref| + 2e-4) <= 1, as the other tests
                   row=float(np.max(np.abs(out["row_loss"].cpu().numpy() - ref["row_loss"]) /
                                    (5e-3 * np.abs(ref["row_loss"]) + 2e-4))),
                   lse=float(np.max(np.abs(out["lse_s"].cpu().numpy() - ref["lse_s"]))),
                   dH=float(np.max(np.abs(out["dH"].double().cpu().numpy() - ref["dH"]))),
                   dH_scale=float(np.max(np.abs(ref["dH"]))),
                   dW=float(np.max(np.abs(dW - ref["dW"][v0:v1]))),
                   dW_scale=float(np.max(np.abs(ref["dW"]))))
        q.put(res)
    except Exception as e:  # report instead of leaving the parent waiting
        q.put(dict(rank=rank, error=repr(e)))
    finally:
        dist.destroy_process_group()


def test_two_processes_over_gloo_on_one_gpu():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_two_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in res:
        assert "error" not in r, r
        assert r["status"] == 0, r
        assert abs(r["loss"] - r["ref_loss"]) <= LOSS_RTOL * abs(r["ref_loss"]), r
        assert r["row"] <= 1.0 and r["lse"] <= 1e-4, r
        assert r["dH"] <= GRAD_FRAC * r["dH_scale"], r
        assert r["dW"] <= GRAD_FRAC * r["dW_scale"], r


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_hidden_shards_with_every_option(dtype):
    """Teacher-hidden shards with a per-token temperature, a mask, reverse-KL
    mixing, several chunks and dW accumulation on top of existing values."""
    w = _hidden(dtype=dtype, seed=40)
    g = torch.Generator().manual_seed(40)
    w.T = (0.6 + 2.0 * torch.rand(w.N, generator=g)).to(torch.float32).cuda()
    kw = dict(_kw(w, chunk=64), reverse_weight=0.4)
    Wt = kw.pop("Wt")
    shards = [(0, 700), (700, 2048), (2048, 3001)]
    base = torch.randn(w.W.shape, generator=g).cuda()
    passes = [vp.ShardPass(w.H, w.W[a:b], v_begin=a, V_total=w.V, Wt=Wt[a:b],
                           dW=base[a:b].clone(), accumulate_dW=True, want_row_loss=True,
                           want_lse=True, **kw) for a, b in shards]
    for k in range(len(passes[0].chunks)):
        st = torch.cat([s.fwd_chunk(k) for s in passes])
        sums = torch.cat([s.mid_chunk(k, st, 3, r) for r, s in enumerate(passes)])
        for r, s in enumerate(passes):
            s.bwd_chunk(k, st, 3, r, 0.9, sums)
    ref = _oracle(w, reverse_weight=0.4, grad_loss=0.9)
    loss = float(sum(s.loss for s in passes))
    assert abs(loss - ref["loss"]) <= LOSS_RTOL * abs(ref["loss"])
    row = sum(s.row_loss for s in passes).cpu().numpy()
    np.testing.assert_allclose(row, ref["row_loss"], rtol=5e-3, atol=2e-4)
    dH32 = sum(s.dH32 for s in passes)
    _check_grad(passes[0].cast_dH(dH32), ref["dH"], "dH")
    dW = torch.cat([s.dW for s in passes]) - base
    _check_grad(dW, ref["dW"], "dW")
    assert all(ops.status(s.ws) == 0 for s in passes)
