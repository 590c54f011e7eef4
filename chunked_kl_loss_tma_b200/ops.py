"""Torch-facing calls of the fused, chunked distillation KL loss.

PyTorch supplies device memory and the current stream; every step of the loss
runs in libchunkedkl.so through its C ABI (see include/chunked_kl.h for what
each call computes, argument layouts and error behaviour).

    out = kl_fwd_bwd(H, W, topk_idx=idx, topk_logit=val, teacher_lse=lse, T=1.0)
    out["loss"], out["dH"], out["dW"]

    loss = fused_kl_loss(H, W, topk_idx=idx, topk_logit=val)   # autograd
    loss.backward()                                            # H.grad, W.grad
"""
from __future__ import annotations

import torch

from . import _lib as L

_DT = {torch.bfloat16: L.KL_DTYPE_BF16, torch.float32: L.KL_DTYPE_F32}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype=None, device=None, shape=None):
    """Check a tensor argument (None passes).  The C ABI takes bare pointers and
    cannot see sizes, so every shape the kernels rely on is checked here."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _workspace(ws, device):
    """A caller's workspace: a contiguous device tensor; its size in bytes (the
    library checks it against kl_workspace_bytes)."""
    _need(ws, "workspace", device=device)
    return ws.numel() * ws.element_size()


def make_problem(H, W, *, T=1.0, mask=None, topk_idx=None, topk_logit=None, teacher_lse=None,
                 Ht=None, Wt=None, chunk_tokens=0, normalizer=0.0, reverse_weight=0.0,
                 v_begin=0, V_total=0, keep_last_chunk=False, fuse_dlogits=False):
    """Fill a kl_problem from tensors.  Returns (problem, tensors kept alive).
    T: a number, or a float32 tensor [N] of per-token temperatures.
    v_begin, V_total: W (and Wt) are rows [v_begin, v_begin + V) of a V_total-row
    head (vocabulary-parallel calls only).
    keep_last_chunk: kl_fwd leaves the last chunk's logits in its workspace for a
    following kl_bwd on the same workspace and inputs (no recompute of that
    chunk).
    fuse_dlogits: kl_fwd_bwd / kl_vp_* form dS inside the dH contraction (bf16
    top-K) instead of by a pass over the logit chunk."""
    if not isinstance(H, torch.Tensor) or not H.is_cuda:
        raise ValueError("H must be a CUDA tensor")
    dev = H.device
    if H.dtype not in _DT:
        raise TypeError("H must be bfloat16 or float32")
    _need(H, "H", H.dtype, dev)
    _need(W, "W", H.dtype, dev)
    if H.dim() != 2 or W.dim() != 2 or H.shape[1] != W.shape[1]:
        raise ValueError("H must be [N, d] and W [V, d]")
    if mask is not None and mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    _need(mask, "mask", torch.uint8, dev, shape=(H.shape[0],))
    p = L.KLProblem()
    p.N, p.d = H.shape
    p.V = W.shape[0]
    p.dtype = _DT[H.dtype]
    p.H, p.W, p.mask = _ptr(H), _ptr(W), _ptr(mask)
    T_row = None
    if isinstance(T, torch.Tensor):
        T_row = _need(T, "T", torch.float32, dev)
        if T_row.shape != (H.shape[0],):
            raise ValueError("a per-token T must be [N]")
        T = 1.0
    p.T = float(T)
    p.T_row = _ptr(T_row)
    p.chunk_tokens = int(chunk_tokens)
    p.normalizer = float(normalizer)
    p.reverse_weight = float(reverse_weight)
    p.v_begin = int(v_begin)
    p.V_total = int(V_total)
    p.keep_last_chunk = 1 if keep_last_chunk else 0
    p.fuse_dlogits = 1 if fuse_dlogits else 0
    keep = [H, W, mask, T_row]
    if Ht is not None:
        _need(Ht, "Ht", H.dtype, dev)
        _need(Wt, "Wt", H.dtype, dev)
        if Ht.shape[0] != H.shape[0] or Wt.shape[0] != W.shape[0] or Ht.shape[1] != Wt.shape[1]:
            raise ValueError("Ht must be [N, d_t] and Wt [V, d_t]")
        p.teacher = L.KL_TEACHER_HIDDEN
        p.d_t = Ht.shape[1]
        p.Ht, p.Wt = _ptr(Ht), _ptr(Wt)
        keep += [Ht, Wt]
    else:
        if topk_idx is None or topk_logit is None:
            raise ValueError("give either topk_idx/topk_logit or Ht/Wt")
        _need(topk_idx, "topk_idx", torch.int32, dev)
        _need(topk_logit, "topk_logit", torch.float32, dev)
        _need(teacher_lse, "teacher_lse", torch.float32, dev, shape=(H.shape[0],))
        if topk_idx.shape != topk_logit.shape or topk_idx.shape[0] != H.shape[0]:
            raise ValueError("topk_idx and topk_logit must both be [N, K]")
        p.teacher = L.KL_TEACHER_TOPK
        p.K = topk_idx.shape[1]
        p.topk_idx, p.topk_logit, p.teacher_lse = (_ptr(topk_idx), _ptr(topk_logit),
                                                   _ptr(teacher_lse))
        keep += [topk_idx, topk_logit, teacher_lse]
    return p, keep


def workspace_bytes(problem, entry):
    n = L.kl_workspace_bytes(problem, entry)
    if n == 0:
        raise ValueError("invalid problem (kl_workspace_bytes returned 0)")
    return n


def alloc_workspace(problem, entry, device):
    return torch.empty(workspace_bytes(problem, entry), dtype=torch.uint8, device=device)


def _stream(device):
    return torch.cuda.current_stream(device).cuda_stream


def kl_fwd_bwd(H, W, *, grad_loss=1.0, dW=None, accumulate_dW=False, want_row_loss=False,
               workspace=None, **kw):
    """Fused forward + backward.  Returns dict(loss, row_loss, dH, dW)."""
    p, keep = make_problem(H, W, **kw)
    dev = H.device
    ws = workspace if workspace is not None else alloc_workspace(p, L.KL_ENTRY_FWD_BWD, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    row_loss = torch.empty(H.shape[0], dtype=torch.float32, device=dev) if want_row_loss else None
    dH = torch.empty_like(H)
    if dW is None:
        dW = torch.empty(W.shape, dtype=torch.float32, device=dev)
        accumulate_dW = False
    _need(dW, "dW", torch.float32, dev, shape=W.shape)
    L.check(L.kl_fwd_bwd(p, ws.data_ptr(), _workspace(ws, dev), grad_loss, loss.data_ptr(),
                         _ptr(row_loss), dH.data_ptr(), dW.data_ptr(), accumulate_dW,
                         _stream(dev)), "kl_fwd_bwd")
    return dict(loss=loss, row_loss=row_loss, dH=dH, dW=dW, workspace=ws)


def kl_fwd(H, W, *, workspace=None, want_row_loss=True, **kw):
    """Forward only.  Returns dict(loss, lse_s, lse_t, row_loss)."""
    p, keep = make_problem(H, W, **kw)
    dev = H.device
    ws = workspace if workspace is not None else alloc_workspace(p, L.KL_ENTRY_FWD, dev)
    N = H.shape[0]
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse_s = torch.empty(N, dtype=torch.float32, device=dev)
    lse_t = torch.empty(N, dtype=torch.float32, device=dev) if kw.get("Ht") is not None else None
    row_loss = torch.empty(N, dtype=torch.float32, device=dev) if want_row_loss else None
    L.check(L.kl_fwd(p, ws.data_ptr(), _workspace(ws, dev), loss.data_ptr(), lse_s.data_ptr(),
                     _ptr(lse_t), _ptr(row_loss), _stream(dev)), "kl_fwd")
    return dict(loss=loss, lse_s=lse_s, lse_t=lse_t, row_loss=row_loss, workspace=ws)


def kl_bwd(H, W, lse_s, lse_t=None, *, grad_loss=None, dW=None, accumulate_dW=False,
           workspace=None, **kw):
    """Backward with logits recomputed per chunk.  grad_loss: device scalar
    tensor (default 1).  Returns dict(dH, dW)."""
    if kw.get("keep_last_chunk") and workspace is None:
        raise ValueError("keep_last_chunk: pass the workspace of the kl_fwd call")
    p, keep = make_problem(H, W, **kw)
    dev = H.device
    ws = workspace if workspace is not None else alloc_workspace(p, L.KL_ENTRY_BWD, dev)
    if grad_loss is None:
        grad_loss = torch.ones((), dtype=torch.float32, device=dev)
    grad_loss = _need(grad_loss.to(torch.float32).reshape(()).contiguous(), "grad_loss",
                      torch.float32, dev)
    N = H.shape[0]
    _need(lse_s, "lse_s", torch.float32, dev, shape=(N,))
    if p.teacher == L.KL_TEACHER_HIDDEN and lse_t is None:
        raise ValueError("lse_t (from kl_fwd) is required in the teacher-hidden mode")
    _need(lse_t, "lse_t", torch.float32, dev, shape=(N,))
    dH = torch.empty_like(H)
    if dW is None:
        dW = torch.empty(W.shape, dtype=torch.float32, device=dev)
        accumulate_dW = False
    _need(dW, "dW", torch.float32, dev, shape=W.shape)
    L.check(L.kl_bwd(p, ws.data_ptr(), _workspace(ws, dev), lse_s.data_ptr(), _ptr(lse_t),
                     grad_loss.data_ptr(), dH.data_ptr(), dW.data_ptr(), accumulate_dW,
                     _stream(dev)), "kl_bwd")
    return dict(dH=dH, dW=dW, workspace=ws)


def status(workspace):
    """Synchronise and return the device-side status word of a workspace."""
    return L.kl_status(workspace.data_ptr(), _stream(workspace.device))


class _FusedKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, kw):
        out = kl_fwd(H, W, want_row_loss=False, **kw)
        ctx.save_for_backward(H, W, out["lse_s"], out["lse_t"] if out["lse_t"] is not None
                              else out["lse_s"])
        ctx.kw = kw
        ctx.hidden = out["lse_t"] is not None
        # with keep_last_chunk the workspace carries the last chunk's logits to
        # the backward (autograd refuses a backward whose H or W changed in place)
        ctx.ws = out["workspace"] if kw.get("keep_last_chunk") else None
        return out["loss"]

    @staticmethod
    def backward(ctx, g):
        H, W, lse_s, lse_t = ctx.saved_tensors
        out = kl_bwd(H, W, lse_s, lse_t if ctx.hidden else None, grad_loss=g.reshape(()),
                     workspace=ctx.ws, **ctx.kw)
        ctx.ws = None
        return out["dH"], out["dW"].to(W.dtype), None


def fused_kl_loss(H, W, *, keep_last_chunk=True, **kw):
    """Differentiable loss (w.r.t. H and W) via kl_fwd / kl_bwd.

    keep_last_chunk (default): the forward's last chunk of logits (one chunk,
    at most chunk_tokens x V values) stays allocated until the backward, which
    then recomputes every chunk but that one -- none when N <= chunk_tokens.
    False: the backward recomputes every chunk and nothing is held between the
    two passes beyond the per-row log-sum-exps."""
    return _FusedKL.apply(H, W, dict(kw, keep_last_chunk=keep_last_chunk))
