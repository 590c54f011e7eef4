"""Parity at the benchmark configurations' full sizes, in the launch
configuration bench.py times (default 4096-token chunks, 2-CTA tiles, split-K
dH), against the fp64 oracle.

Outputs the oracle can compute one by one are compared element by element on
sampled rows (first and last rows, chunk boundaries, masked rows, random
rows): row loss, lse and dH rows, each sampled row evaluated by the oracle as a
problem of its own with the full problem's normaliser.  Up to N=65536 the
oracle also makes its full pass over every row, which gives the loss itself,
every row's loss, and dW on sampled vocabulary rows -- among them the rows the
teacher's mass concentrates on (the most frequent cached ids, or the teacher's
most frequent argmax in the teacher-hidden mode).  At N=262144, where a full
fp64 pass takes too long, the loss is checked as the mean of the row losses and
dW through identities that hold at any size: every dS row sums to zero
(sum_j (m p_s,j - q_j) = m - m = 0, and sum_j (p_s,j - p_t,j) = 0), so
sum_j dW_j = 0; and <dW, W> = <dH, H> = sum_{n,j} dS_nj s_nj.  The identities
are checked everywhere as extra checks.

Tolerances as in test_parity_gpu.py: loss relative error <= 1e-3; gradient
max-abs error <= 2e-2 * max|oracle gradient| (over the sampled entries)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _rows(N, mask, n_random=24, seed=0):
    rng = np.random.default_rng(seed)
    cand = {0, 1, N - 1, N - 2}
    for b in range(4096, N, 4096):  # chunk boundaries
        cand.update({b - 1, b})
    cand.update(rng.choice(N, size=min(n_random, N), replace=False).tolist())
    if mask is not None:
        masked = np.nonzero(mask.cpu().numpy() == 0)[0]
        if len(masked):
            cand.update(rng.choice(masked, size=min(4, len(masked)), replace=False).tolist())
    return np.array(sorted(c for c in cand if 0 <= c < N))


def _kw(w):
    kw = dict(T=w.T, mask=w.mask)
    if w.mode == "topk":
        kw.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        kw.update(Ht=w.Ht, Wt=w.Wt)
    return kw


def _oracle_rows(w, rows, n_valid, g=1.0, reverse_weight=0.0):
    r = torch.as_tensor(rows, device=w.H.device)
    args = dict(T=w.T, mode=w.mode, grad_loss=g, normalizer=n_valid, want_dW=False,
                mask=None if w.mask is None else w.mask[r], reverse_weight=reverse_weight)
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx[r], topk_logit=w.topk_logit[r],
                    teacher_lse=None if w.teacher_lse is None else w.teacher_lse[r])
    else:
        args.update(Ht=w.Ht[r], Wt=w.Wt)
    return oracle.kl_loss(w.H[r], w.W, **args)


def _check_rows(w, out, rows, n_valid):
    ref = _oracle_rows(w, rows, n_valid)
    r = torch.as_tensor(rows, device=w.H.device)
    rl = out["row_loss"][r].double().cpu().numpy()
    scale = max(np.max(np.abs(ref["row_loss"])), 1e-12)
    assert np.max(np.abs(rl - ref["row_loss"])) <= 2e-3 * scale, "row loss"
    dH = out["dH"][r].double().cpu().numpy()
    err = np.max(np.abs(dH - ref["dH"]))
    assert err <= 2e-2 * np.max(np.abs(ref["dH"])), f"dH rows: {err}"
    if w.mask is not None:
        m = w.mask[r].cpu().numpy() == 0
        assert np.all(rl[m] == 0) and np.all(dH[m] == 0), "masked rows"
    return ref


def _identities(w, out):
    dW = out["dW"]
    colsum = dW.double().sum(0)
    assert colsum.abs().max().item() <= 1e-2 * dW.double().abs().sum(0).max().item() + 1e-30
    a = (dW.double() * w.W.double()).sum().item()
    b = (out["dH"].double() * w.H.double()).sum().item()
    assert abs(a - b) <= 1e-2 * max(abs(a), abs(b)), (a, b)
    assert abs(a) > 0


def _vocab_rows(w, n_hot=24, n_random=16, seed=1):
    """Vocabulary rows for the dW check: the ids that carry the teacher's mass
    most often (the cached ids, or the teacher's argmax computed with a plain
    torch matmul), random rows, and the first and last rows."""
    if w.mode == "topk":
        ids = w.topk_idx[:, :4].reshape(-1)
        ids = ids[ids >= 0]
    else:
        ids = torch.cat([(w.Ht[i:i + 2048].float() @ w.Wt.float().T).argmax(1)
                         for i in range(0, w.N, 2048)])
    counts = torch.bincount(ids.long(), minlength=w.V)
    hot = torch.topk(counts, n_hot).indices.cpu().numpy()
    rnd = np.random.default_rng(seed).choice(w.V, n_random, replace=False)
    return np.unique(np.concatenate([hot, rnd, [0, w.V - 1]]))


def _full_oracle_pass(w, out, n_valid, reverse_weight=0.0):
    """The oracle over every row: the loss (relative error <= 1e-3), every
    row's loss, and dW on sampled vocabulary rows (max-abs error <= 2e-2 of the
    largest oracle entry)."""
    vrows = _vocab_rows(w)
    args = dict(T=w.T, mode=w.mode, mask=w.mask, want_dH=False, vocab_rows=vrows,
                reverse_weight=reverse_weight)
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    ref = oracle.kl_loss(w.H, w.W, **args)
    assert ref["n_valid"] == n_valid
    assert abs(out["loss"].item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]), \
        (out["loss"].item(), ref["loss"])
    rl = out["row_loss"].double().cpu().numpy()
    assert np.max(np.abs(rl - ref["row_loss"])) <= 2e-3 * np.max(np.abs(ref["row_loss"]))
    dW = out["dW"][torch.as_tensor(vrows, device=out["dW"].device)].double().cpu().numpy()
    err = np.max(np.abs(dW - ref["dW"]))
    assert err <= 2e-2 * np.max(np.abs(ref["dW"])), f"dW rows: {err}"
    return ref


def _loss_is_mean_of_rows(out, n_valid):
    mean = out["row_loss"].double().sum().item() / n_valid
    assert abs(out["loss"].item() - mean) <= 1e-5 * abs(mean)


def test_offline_topk_4096_full_oracle_pass():
    w = wl.offline_topk(device="cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    assert ops.status(out["workspace"]) == 0
    n_valid = w.N
    rows = _rows(w.N, None)
    _check_rows(w, out, rows, n_valid)
    _loss_is_mean_of_rows(out, n_valid)
    _full_oracle_pass(w, out, n_valid)
    _identities(w, out)


def test_offline_topk_4096_fused_dlogits():
    """The bench workload with dS formed inside the dH contraction: the oracle's
    sampled rows, the identities and the separate-pass result."""
    w = wl.offline_topk(device="cuda", seed=9)
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, fuse_dlogits=True, **_kw(w))
    assert ops.status(out["workspace"]) == 0
    rows = _rows(w.N, None, n_random=16, seed=9)
    _check_rows(w, out, rows, w.N)
    _loss_is_mean_of_rows(out, w.N)
    _identities(w, out)
    # The two paths round dS differently (the fused one rounds its bf16 scale and
    # then the product); both are held to the gradient tolerance against the
    # oracle above, and to the same bound against each other.
    plain = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    assert torch.equal(out["loss"], plain["loss"])
    for k in ("dH", "dW"):
        a, c = out[k].double(), plain[k].double()
        assert (a - c).abs().max().item() <= 2e-2 * c.abs().max().item(), k


def test_offline_topk_4096_split_forward_backward():
    """kl_fwd then kl_bwd (backward recomputes the logits and forms dS in the
    GEMM epilogue) against the oracle's sampled rows and the fused path."""
    w = wl.offline_topk(device="cuda", seed=5)
    kw = _kw(w)
    f = ops.kl_fwd(w.H, w.W, **kw)
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], **kw)
    assert ops.status(f["workspace"]) == 0 and ops.status(b["workspace"]) == 0
    fused = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    out = dict(row_loss=f["row_loss"], dH=b["dH"], dW=b["dW"], loss=f["loss"])
    rows = _rows(w.N, None, n_random=16, seed=5)
    _check_rows(w, out, rows, w.N)
    _loss_is_mean_of_rows(out, w.N)
    _identities(w, out)
    assert abs(f["loss"].item() - fused["loss"].item()) <= 1e-5 * abs(fused["loss"].item())
    for k in ("dH", "dW"):
        a, c = b[k].double(), fused[k].double()
        assert (a - c).abs().max().item() <= 2e-2 * c.abs().max().item(), k


def test_full_vocab_8192_teacher_hidden():
    w = wl.full_vocab(device="cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    assert ops.status(out["workspace"]) == 0
    rows = _rows(w.N, None, n_random=16)
    _check_rows(w, out, rows, w.N)
    _loss_is_mean_of_rows(out, w.N)
    _full_oracle_pass(w, out, w.N)
    _identities(w, out)
    # the split forward gives the same loss and the teacher lse of the oracle
    f = ops.kl_fwd(w.H, w.W, **_kw(w))
    ref = _oracle_rows(w, rows, w.N)
    r = torch.as_tensor(rows, device="cuda")
    np.testing.assert_allclose(f["lse_t"][r].double().cpu().numpy(), ref["lse_t"], rtol=1e-5)
    assert abs(f["loss"].item() - out["loss"].item()) <= 1e-4 * abs(out["loss"].item())


def test_full_vocab_8192_mixed_kl():
    """Forward/reverse mixing (beta = 0.5) at the teacher-hidden configuration."""
    w = wl.full_vocab(device="cuda", seed=6)
    kw = dict(_kw(w), reverse_weight=0.5)
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    assert ops.status(out["workspace"]) == 0
    rows = _rows(w.N, None, n_random=12, seed=6)
    ref = _oracle_rows(w, rows, w.N, reverse_weight=0.5)
    r = torch.as_tensor(rows, device="cuda")
    rl = out["row_loss"][r].double().cpu().numpy()
    assert np.max(np.abs(rl - ref["row_loss"])) <= 2e-3 * np.max(np.abs(ref["row_loss"]))
    dH = out["dH"][r].double().cpu().numpy()
    assert np.max(np.abs(dH - ref["dH"])) <= 2e-2 * np.max(np.abs(ref["dH"]))
    _loss_is_mean_of_rows(out, w.N)
    _identities(w, out)


def test_packed_long_32768_masked():
    w = wl.packed_long(device="cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    assert ops.status(out["workspace"]) == 0
    n_valid = int(w.mask.sum().item())
    assert n_valid == w.N - round(0.05 * w.N)
    rows = _rows(w.N, w.mask)
    _check_rows(w, out, rows, n_valid)
    _loss_is_mean_of_rows(out, n_valid)
    _full_oracle_pass(w, out, n_valid)
    _identities(w, out)


@pytest.mark.parametrize("N", [4096, 16384, 65536, 262144])
def test_scaling_sweep_rows_and_flat_memory(N):
    w = wl.scaling(N, device="cuda")
    torch.cuda.empty_cache()
    kw = _kw(w)
    p, keep = ops.make_problem(w.H, w.W, **kw)
    ws_bytes = ops.workspace_bytes(p, 2)
    p4, _ = ops.make_problem(w.H[:4096], w.W, **dict(kw, topk_idx=w.topk_idx[:4096],
                                                      topk_logit=w.topk_logit[:4096],
                                                      teacher_lse=w.teacher_lse[:4096]))
    # extra memory is one chunk's buffers plus O(N) row statistics, never O(N V)
    assert ws_bytes - ops.workspace_bytes(p4, 2) <= 8 * (N - 4096) + 4096
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    torch.cuda.synchronize()
    outputs = out["dH"].numel() * 2 + out["dW"].numel() * 4 + N * 4 + 4
    extra = torch.cuda.max_memory_allocated() - base - outputs
    assert extra <= ws_bytes + (16 << 20), (extra, ws_bytes)  # allocator rounding
    assert ops.status(out["workspace"]) == 0
    rows = _rows(N, None, n_random=12, seed=N)
    _check_rows(w, out, rows, N)
    _loss_is_mean_of_rows(out, N)
    if N <= 65536:
        _full_oracle_pass(w, out, N)
    _identities(w, out)


@pytest.mark.parametrize("cfg,P", [("offline_topk", 8), ("full_vocab", 4)])
def test_vocabulary_parallel_full_size(cfg, P):
    """The head split over P vocabulary shards (emulated one after another on
    one GPU, each shard with its own workspace and the bench's chunking): the
    oracle's sampled rows, the identities, and agreement with the whole-head
    fused call."""
    from chunked_kl_loss_tma_b200 import vocab_parallel as vp

    w = wl.offline_topk(device="cuda", seed=7) if cfg == "offline_topk" else \
        wl.full_vocab(device="cuda", seed=8)
    kw = _kw(w)
    Wt = kw.pop("Wt", None)
    out = vp.emulate(w.H, w.W, P, Wt=Wt, want_row_loss=True, want_lse=True, **kw)
    assert all(ops.status(ws) == 0 for ws in out["workspaces"])
    del out["workspaces"]
    rows = _rows(w.N, None, n_random=12, seed=P)
    ref = _check_rows(w, out, rows, w.N)
    r = torch.as_tensor(rows, device="cuda")
    np.testing.assert_allclose(out["lse_s"][r].double().cpu().numpy(), ref["lse_s"], rtol=1e-5)
    _loss_is_mean_of_rows(out, w.N)
    _identities(w, out)
    whole = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    assert abs(out["loss"].item() - whole["loss"].item()) <= 1e-5 * abs(whole["loss"].item())
    for k in ("dH", "dW"):
        a, c = out[k].double(), whole[k].double()
        assert (a - c).abs().max().item() <= 1e-2 * c.abs().max().item(), k
