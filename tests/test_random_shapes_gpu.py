"""Seeded random problems through the CUDA path against the fp64 oracle.

Each case draws its sizes and options from one seed: the token count N, the
widths d and d_t (multiples of 8), the vocabulary V (often not a multiple of 8
or of the 256-column tile), the cache width K (up to V), the teacher mode, bf16
or fp32 inputs, a scalar or per-token temperature, a random mask, the chunk size
(down to chunks of 1 and 3 rows), partial mass or renormalised teacher
probabilities, a reverse-KL weight in the teacher-hidden mode, and the entry:
the fused pass (with or without dS formed inside the dH contraction) or kl_fwd
followed by kl_bwd (with or without the kept last chunk).

A second set of seeds runs the vocabulary-parallel form (`vocab_parallel.emulate`,
the head cut into 2 to 4 shards at random rows) against the oracle on the
whole problem.

Tolerances as in the other parity tests: loss relative error <= 1e-3 (plus 1e-6
absolute, for losses that are 0), gradients max-abs error <= 2e-2 * max|oracle
gradient|."""
import os

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# Seeds per family; a larger sweep: KL_RANDOM_CASES=1248 KL_RANDOM_WIDE_CASES=60
# KL_RANDOM_VP_CASES=80 python -m pytest tests/test_random_shapes_gpu.py
CASES = int(os.environ.get("KL_RANDOM_CASES", 48))


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    mode = "hidden" if rng.random() < 0.35 else "topk"
    dtype = torch.float32 if rng.random() < 0.2 else torch.bfloat16
    N = int(rng.integers(1, 700))
    d = 8 * int(rng.integers(1, 70))
    V = int(rng.choice([int(rng.integers(1, 300)), int(rng.integers(300, 9000))]))
    K = int(rng.integers(1, min(V, 96) + 1))
    d_t = 8 * int(rng.integers(1, 40))
    per_token = rng.random() < 0.3
    T = float(rng.uniform(0.5, 3.0))
    chunk = int(rng.choice([0, 64, 200, 512, 1, 3]))
    if chunk in (1, 3):  # many one- or three-row chunks: keep the count of launches small
        N = min(N, 40)
    masked = rng.random() < 0.5
    partial = rng.random() < 0.6
    beta = float(rng.choice([0.0, 0.0, 0.3, 1.0])) if mode == "hidden" else 0.0
    entry = str(rng.choice(["fused", "fused", "split", "split_keep"]))
    fuse = bool(mode == "topk" and dtype == torch.bfloat16 and entry == "fused" and
                rng.random() < 0.5)
    g = float(rng.uniform(0.3, 2.0))
    Tr = None
    if per_token:
        Tr = torch.from_numpy(rng.uniform(0.5, 3.0, size=N).astype(np.float32))
    w_std = float(rng.uniform(0.03, 0.3))
    if mode == "topk":
        w = wl.make_topk(f"rand{seed}", N=N, d=d, V=V, K=K, d_t=d_t, T=Tr if per_token else T,
                         dtype=dtype, w_std=w_std, tw_std=float(rng.uniform(0.05, 0.3)),
                         seed=2000 + seed, partial_mass=partial)
    else:
        w = wl.make_hidden(f"randh{seed}", N=N, d=d, d_t=d_t, V=V, T=Tr if per_token else T,
                           dtype=dtype, w_std=w_std, tw_std=float(rng.uniform(0.05, 0.3)),
                           seed=2000 + seed)
    if masked:
        w.mask = torch.from_numpy((rng.random(N) > 0.25).astype(np.uint8))
    opts = dict(chunk=chunk, beta=beta, entry=entry, fuse=fuse, g=g)
    return w.to("cuda"), opts


def _kw(w, opts):
    kw = dict(T=w.T, mask=w.mask, chunk_tokens=opts["chunk"], reverse_weight=opts["beta"])
    if w.mode == "topk":
        kw.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        kw.update(Ht=w.Ht, Wt=w.Wt)
    return kw


@pytest.mark.parametrize("seed", range(CASES))
def test_random_problem_matches_oracle(seed):
    w, o = _draw(seed)
    kw = _kw(w, o)
    if o["entry"] == "fused":
        out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=o["g"], fuse_dlogits=o["fuse"], **kw)
        loss, dH, dW, wss = out["loss"], out["dH"], out["dW"], [out["workspace"]]
    else:
        keep = o["entry"] == "split_keep"
        f = ops.kl_fwd(w.H, w.W, keep_last_chunk=keep, **kw)
        b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"],
                       grad_loss=torch.full((), o["g"], device="cuda"),
                       workspace=f["workspace"] if keep else None, keep_last_chunk=keep, **kw)
        loss, dH, dW, wss = f["loss"], b["dH"], b["dW"], [f["workspace"], b["workspace"]]
    assert all(ops.status(ws) == 0 for ws in wss)
    args = dict(T=w.T, mask=w.mask, mode=w.mode, grad_loss=o["g"], reverse_weight=o["beta"])
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    ref = oracle.kl_loss(w.H, w.W, **args)
    case = f"seed {seed}: N={w.N} d={w.d} V={w.V} {w.mode} {w.dtype} {o}"
    assert abs(loss.item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]) + 1e-6, \
        (case, loss.item(), ref["loss"])
    for name, got in (("dH", dH), ("dW", dW)):
        r = ref[name]
        err = np.max(np.abs(got.double().cpu().numpy() - r))
        assert err <= 2e-2 * np.max(np.abs(r)) + 1e-6, (case, name, err, np.max(np.abs(r)))


VP_CASES = int(os.environ.get("KL_RANDOM_VP_CASES", 16))


def _draw_vp(seed):
    """A random problem for the vocabulary-parallel form: as _draw, with the head
    cut into P = 2..4 shards at random rows (boundaries inside tiles, shards of
    a few rows among them)."""
    rng = np.random.default_rng(7000 + seed)
    mode = "hidden" if rng.random() < 0.45 else "topk"
    dtype = torch.float32 if rng.random() < 0.2 else torch.bfloat16
    N = int(rng.integers(1, 400))
    d = 8 * int(rng.integers(1, 40))
    P = int(rng.integers(2, 5))
    V = int(rng.integers(P + 1, 6000))
    cuts = np.sort(rng.choice(np.arange(1, V), size=P - 1, replace=False))
    bounds = [0] + [int(c) for c in cuts] + [V]
    shards = [(bounds[i], bounds[i + 1]) for i in range(P)]
    K = int(rng.integers(1, min(V, 64) + 1))
    d_t = 8 * int(rng.integers(1, 24))
    T = float(rng.uniform(0.5, 3.0))
    Tr = torch.from_numpy(rng.uniform(0.5, 3.0, size=N).astype(np.float32)) \
        if rng.random() < 0.3 else None
    chunk = int(rng.choice([0, 64, 200]))
    beta = float(rng.choice([0.0, 0.4, 1.0])) if mode == "hidden" else 0.0
    fuse = bool(mode == "topk" and dtype == torch.bfloat16 and rng.random() < 0.4)
    g = float(rng.uniform(0.3, 2.0))
    w_std = float(rng.uniform(0.03, 0.3))
    if mode == "topk":
        w = wl.make_topk(f"vp{seed}", N=N, d=d, V=V, K=K, d_t=d_t,
                         T=Tr if Tr is not None else T, dtype=dtype, w_std=w_std,
                         tw_std=float(rng.uniform(0.05, 0.3)), seed=8000 + seed,
                         partial_mass=rng.random() < 0.6)
    else:
        w = wl.make_hidden(f"vph{seed}", N=N, d=d, d_t=d_t, V=V,
                           T=Tr if Tr is not None else T, dtype=dtype, w_std=w_std,
                           tw_std=float(rng.uniform(0.05, 0.3)), seed=8000 + seed)
    if rng.random() < 0.5:
        w.mask = torch.from_numpy((rng.random(N) > 0.25).astype(np.uint8))
    return w.to("cuda"), dict(shards=shards, chunk=chunk, beta=beta, fuse=fuse, g=g)


@pytest.mark.parametrize("seed", range(VP_CASES))
def test_random_vocabulary_shards_match_oracle(seed):
    from chunked_kl_loss_tma_b200 import vocab_parallel as vp

    w, o = _draw_vp(seed)
    kw = _kw(w, o)
    Wt = kw.pop("Wt", None)
    out = vp.emulate(w.H, w.W, len(o["shards"]), shards=o["shards"], grad_loss=o["g"], Wt=Wt,
                     fuse_dlogits=o["fuse"], **kw)
    assert all(ops.status(ws) == 0 for ws in out["workspaces"])
    args = dict(T=w.T, mask=w.mask, mode=w.mode, grad_loss=o["g"], reverse_weight=o["beta"])
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    ref = oracle.kl_loss(w.H, w.W, **args)
    case = f"vp seed {seed}: N={w.N} d={w.d} V={w.V} {w.mode} {w.dtype} {o}"
    assert abs(out["loss"].item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]) + 1e-6, \
        (case, out["loss"].item(), ref["loss"])
    for name in ("dH", "dW"):
        r = ref[name]
        err = np.max(np.abs(out[name].double().cpu().numpy() - r))
        assert err <= 2e-2 * np.max(np.abs(r)) + 1e-6, (case, name, err, np.max(np.abs(r)))


WIDE_CASES = int(os.environ.get("KL_RANDOM_WIDE_CASES", 8))


@pytest.mark.parametrize("seed", range(WIDE_CASES))
def test_random_wide_problem_matches_oracle(seed):
    """Wide heads (d from 1024 to 4096, many short dW units per CTA pair, V
    rarely a multiple of 256) with the options of _draw; fewer tokens so that
    the oracle stays quick."""
    rng = np.random.default_rng(9000 + seed)
    w, o = _draw(100 + seed)
    masked = w.mask is not None
    d = 8 * int(rng.integers(128, 513))
    N = min(w.N, 300)
    V = min(w.V, 3000)
    base = dict(T=w.T if not torch.is_tensor(w.T) else w.T[:N].cpu(), dtype=w.dtype,
                w_std=0.02, seed=9500 + seed)
    if w.mode == "topk":
        w = wl.make_topk(f"rwide{seed}", N=N, d=d, V=V, K=min(w.K, V), d_t=w.d_t,
                         tw_std=0.05, partial_mass=w.teacher_lse is not None, **base)
    else:
        w = wl.make_hidden(f"rwideh{seed}", N=N, d=d, d_t=w.d_t, V=V, tw_std=0.05, **base)
    if masked:
        w.mask = torch.from_numpy((rng.random(N) > 0.25).astype(np.uint8))
    w = w.to("cuda")
    kw = _kw(w, o)
    if o["entry"] == "fused":
        out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=o["g"], fuse_dlogits=o["fuse"], **kw)
        loss, dH, dW, wss = out["loss"], out["dH"], out["dW"], [out["workspace"]]
    else:
        keep = o["entry"] == "split_keep"
        f = ops.kl_fwd(w.H, w.W, keep_last_chunk=keep, **kw)
        b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"],
                       grad_loss=torch.full((), o["g"], device="cuda"),
                       workspace=f["workspace"] if keep else None, keep_last_chunk=keep, **kw)
        loss, dH, dW, wss = f["loss"], b["dH"], b["dW"], [f["workspace"], b["workspace"]]
    assert all(ops.status(ws) == 0 for ws in wss)
    args = dict(T=w.T, mask=w.mask, mode=w.mode, grad_loss=o["g"], reverse_weight=o["beta"])
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    ref = oracle.kl_loss(w.H, w.W, **args)
    case = f"wide seed {seed}: N={w.N} d={w.d} V={w.V} {w.mode} {w.dtype} {o}"
    assert abs(loss.item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]) + 1e-6, \
        (case, loss.item(), ref["loss"])
    for name, got in (("dH", dH), ("dW", dW)):
        r = ref[name]
        err = np.max(np.abs(got.double().cpu().numpy() - r))
        assert err <= 2e-2 * np.max(np.abs(r)) + 1e-6, (case, name, err, np.max(np.abs(r)))
