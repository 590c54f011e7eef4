"""Plain fp64 CPU oracle for the distillation KL loss over the LM output head.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (``chunked_kl_loss_tma_b200``) never imports it and
shares no code with it: no helpers, no constants, no pre/post-processing.

What it computes, written as the plain definition (no chunking, no fusion, no
online reductions; one fp64 matrix product per logit block as the only library
step):

Source: "Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and a
Fused Chunked KL Loss" (Ryskulov et al.), section-by-section summary page:
  * §1 Introduction, "Fused, chunked KL loss": a forward-KL distillation
    objective whose teacher side is a sparse top-K distribution that keeps
    only part of the probability mass.
  * §3 Types of Knowledge Distillation, "Online distillation": dense teacher
    probabilities against student log-probabilities (forward KL(p_t || p_s)).
  * §3 "Offline distillation": the cache stores the teacher's K most likely
    tokens with probabilities that are not renormalised over those K; the
    student contributes its log-probabilities at the K cached tokens and one
    normaliser per token.
  * §3 "Offline implementations": the reference variant expands the cache
    into a dense teacher distribution over the vocabulary; the dense
    reconstruction below is that check.
And the KDFlow abstract (thelatestinai.com/papers/2603.01875): full-vocabulary
distillation with teacher logits recomputed from the teacher's final hidden
states through a frozen copy of the teacher's output head.

Readings where the pages are silent:
  R1 temperature T divides both student and teacher logits; no T^2 factor.
  R2 partial mass: q_i = exp(t_i/T - lse_t) with lse_t the teacher's full
     vocabulary log-sum-exp at the same T (supplied with the cache); the mass
     term is m * lse_s with m = sum_i q_i, no residual bucket.
     Renormalised (no lse_t supplied): q_i = softmax over the valid cached
     entries of t_i/T.
  R3 reduction: mean over unmasked tokens (normaliser = number of mask=1 rows
     unless the caller passes another normaliser); zero valid rows -> loss 0.
  R4 cache slot with index -1 is empty (contributes nothing); a row with no
     valid slot contributes 0; duplicate or out-of-range indices are errors.
  R5 frozen teacher head: no gradient flows to Ht or Wt.
  R6 KL direction mixing (teacher-hidden mode only): the page's KL-direction
     study (thelatestinai.com/papers/2606.20005, fourth abstract) names
     token-level reverse KL and "KL mixing"; read as the convex combination
     l = (1 - beta) KL(p_t || p_s) + beta KL(p_s || p_t), beta in [0, 1]
     (beta = 0 is the forward KL of the fused-loss paper).  Undefined for a
     top-K cache (the student mass outside the support has no teacher value).
  R7 per-token temperature: the entropy-adaptive KD abstract on page 4
     (thelatestinai.com/papers/2610.07706) adjusts the distillation temperature
     per token; read as T given per row (T_n divides row n's student and
     teacher logits, and its gradient carries 1/T_n).  A scalar T is the same
     value for every row.

Parity pins for every function live in tests/test_oracle_pins.py (closed
forms, hand-derived fixtures in tests/golden/, library KL routines, autograd,
central finite differences, K=V equivalence, dense reconstruction).
"""
from __future__ import annotations

import numpy as np

TOPK = "topk"
HIDDEN = "hidden"


def _f64(x):
    """Exact widening of the caller's values (bf16/fp32 -> fp64 is exact)."""
    if x is None:
        return None
    try:  # torch tensors (bf16 has no numpy dtype: widen through float32)
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


def logsumexp_rows(x):
    """log sum_j exp(x_j) per row, written as max + log sum exp(x - max).

    The shift by the row maximum is an exact identity, not an approximation.
    This is the per-token student normaliser of §3 "Offline distillation"."""
    m = np.max(x, axis=1, keepdims=True)
    return (m + np.log(np.sum(np.exp(x - m), axis=1, keepdims=True)))[:, 0]


def _col(T):
    """Temperature as a column to divide row blocks by (scalar or one per row)."""
    T = np.asarray(T, dtype=np.float64)
    return T if T.ndim == 0 else T[:, None]


def scaled_logits(X, Wh, T):
    """x~ = (X . Wh^T) / T for a block of rows: the output projection of the
    head (§3 "Fused chunked KL": the loss integrates the output projection)
    followed by temperature scaling (readings R1, R7: T scalar or one per
    row).  fp64 matrix product."""
    return (X @ Wh.T) / _col(T)


def teacher_support_probs(topk_idx, topk_logit, T, teacher_lse, V):
    """Teacher probabilities on the cached support (§3 "Offline distillation").

    Returns (idx, q, valid) with q[n, i] the teacher probability of cached
    entry i of row n:
      * partial mass (teacher_lse given): q = exp(t/T - lse_t); the K entries
        keep their unnormalised share of the full distribution (reading R2);
      * renormalised (teacher_lse is None): q = softmax over the row's valid
        entries of t/T.
    Empty slots (index -1) get q = 0 (reading R4)."""
    idx = _i64(topk_idx)
    t = _f64(topk_logit) / _col(T)
    valid = idx >= 0
    if np.any(idx >= V) or np.any(idx < -1):
        raise ValueError("top-K index out of range")
    for n in range(idx.shape[0]):
        row = idx[n][valid[n]]
        if len(np.unique(row)) != len(row):
            raise ValueError(f"duplicate top-K index in row {n}")
    if teacher_lse is not None:
        lse_t = _f64(teacher_lse)
        q = np.where(valid, np.exp(t - lse_t[:, None]), 0.0)
    else:
        tm = np.where(valid, t, -np.inf)
        mx = np.max(tm, axis=1, keepdims=True)
        mx = np.where(np.isfinite(mx), mx, 0.0)
        e = np.where(valid, np.exp(tm - mx), 0.0)
        z = np.sum(e, axis=1, keepdims=True)
        q = np.where(z > 0, e / np.where(z > 0, z, 1.0), 0.0)
    return idx, q, valid


def kl_topk_rows(s_tilde, lse_s, idx, q, valid):
    """Per-row forward KL against the cached support (§1, §3):
        l_n = sum_{i in S_n} q_i * (log q_i - log p_s[idx_i]),
    with log p_s = s~ - lse_s.  0*log 0 = 0."""
    safe = np.where(valid, idx, 0)
    log_ps = np.take_along_axis(s_tilde, safe, axis=1) - lse_s[:, None]
    qlogq = np.where(q > 0, q * np.log(np.where(q > 0, q, 1.0)), 0.0)
    return np.sum(np.where(valid, qlogq - q * log_ps, 0.0), axis=1)


def grad_topk_rows(s_tilde, lse_s, idx, q, valid, T):
    """d l_n / d s (raw logits) for the top-K loss above:
        (m * p_s[j] - q_j * [j in S_n]) / T,   m = sum_i q_i.
    Derivation: d log p_s[k]/d s~_j = [j = k] - p_s[j]; d s~/d s = 1/T."""
    p_s = np.exp(s_tilde - lse_s[:, None])
    m = np.sum(q, axis=1)
    g = m[:, None] * p_s
    rows = np.arange(idx.shape[0])
    for i in range(idx.shape[1]):
        sel = valid[:, i]
        g[rows[sel], idx[sel, i]] -= q[sel, i]
    return g / _col(T)


def kl_full_rows(s_tilde, lse_s, t_tilde, lse_t):
    """Per-row full-vocabulary forward KL (§3 "Online distillation"; KDFlow
    abstract for the recomputed teacher logits):
        l_n = sum_j p_t[j] * (log p_t[j] - log p_s[j])."""
    log_pt = t_tilde - lse_t[:, None]
    log_ps = s_tilde - lse_s[:, None]
    p_t = np.exp(log_pt)
    return np.sum(p_t * (log_pt - log_ps), axis=1)


def grad_full_rows(s_tilde, lse_s, t_tilde, lse_t, T):
    """d l_n / d s (raw logits) for the full KL: (p_s[j] - p_t[j]) / T."""
    return (np.exp(s_tilde - lse_s[:, None]) - np.exp(t_tilde - lse_t[:, None])) / _col(T)


def kl_reverse_rows(s_tilde, lse_s, t_tilde, lse_t):
    """Per-row reverse KL: l_n = sum_j p_s[j] * (log p_s[j] - log p_t[j])."""
    log_pt = t_tilde - lse_t[:, None]
    log_ps = s_tilde - lse_s[:, None]
    p_s = np.exp(log_ps)
    return np.sum(p_s * (log_ps - log_pt), axis=1)


def grad_reverse_rows(s_tilde, lse_s, t_tilde, lse_t, T):
    """d l_n / d s (raw logits) for the reverse KL: p_s[j] (u_j - u_bar) / T with
    u = log p_s - log p_t and u_bar = sum_j p_s[j] u_j.
    Derivation: d/ds~_k sum_j p_s[j] u_j = sum_j p_s[j] ([j=k] - p_s[k]) u_j
    + p_s[k] - p_s[k] sum_j p_s[j] = p_s[k] (u_k - u_bar)."""
    log_ps = s_tilde - lse_s[:, None]
    u = log_ps - (t_tilde - lse_t[:, None])
    p_s = np.exp(log_ps)
    u_bar = np.sum(p_s * u, axis=1, keepdims=True)
    return p_s * (u - u_bar) / _col(T)


def kl_loss(H, W, *, T=1.0, mask=None, mode=TOPK, topk_idx=None, topk_logit=None,
            teacher_lse=None, Ht=None, Wt=None, grad_loss=1.0, normalizer=None,
            rows=None, vocab_rows=None, want_dH=True, want_dW=True, block=256,
            reverse_weight=0.0):
    """The distillation loss L = (1 / n_valid) * sum_{mask_n = 1} l_n and the
    gradients dH = dS . W, dW = dS^T . H of g * L, with dS = g * dL/ds and g
    the incoming gradient of the loss (readings R1-R5).

    rows:        evaluate row quantities (row_loss, lse, dH) only for these
                 token rows (None = all).  Per-row results do not depend on
                 which other rows are evaluated.
    vocab_rows:  rows of dW to return (None = all V).  dW always sums over
                 every token, so it needs all rows' lse.
    normalizer:  divide by this instead of the local unmasked count.
    reverse_weight: beta of reading R6 (teacher-hidden mode only).
    T:           scalar, or one temperature per token row (reading R7).
    block:       rows per fp64 matrix product (memory bound only; every row is
                 an independent computation).

    Returns a dict with loss (only when rows is None), n_valid, row_loss,
    lse_s, lse_t (hidden mode), dH (rows x d), dW (vocab_rows x d)."""
    H = _f64(H)
    W = _f64(W)
    N, d = H.shape
    V = W.shape[0]
    T_all = _f64(T)
    if np.any(T_all <= 0) or (T_all.ndim == 1 and T_all.shape[0] != N) or T_all.ndim > 1:
        raise ValueError("temperature must be > 0 (scalar or one per row)")
    beta = float(reverse_weight)
    if not 0.0 <= beta <= 1.0 or (beta > 0 and mode != HIDDEN):
        raise ValueError("reverse_weight must be in [0, 1] and needs the teacher-hidden mode")
    keep = np.ones(N, dtype=bool) if mask is None else (_i64(mask) != 0)
    n_valid = int(np.sum(keep))
    norm = float(n_valid if normalizer is None else normalizer)
    coef = (grad_loss / norm) if norm > 0 else 0.0

    def T_of(r):
        return T_all if T_all.ndim == 0 else T_all[r]

    if mode == TOPK:
        idx_all, q_all, valid_all = teacher_support_probs(topk_idx, topk_logit, T_all,
                                                          teacher_lse, V)
    elif mode == HIDDEN:
        Ht = _f64(Ht)
        Wt = _f64(Wt)
    else:
        raise ValueError(mode)

    def block_terms(r):
        """Row losses, lse and dS (= coef * dl/ds, zero on masked rows) for
        the token rows r."""
        Tr = T_of(r)
        s = scaled_logits(H[r], W, Tr)
        lse_s = logsumexp_rows(s)
        if mode == TOPK:
            l = kl_topk_rows(s, lse_s, idx_all[r], q_all[r], valid_all[r])
            gr = grad_topk_rows(s, lse_s, idx_all[r], q_all[r], valid_all[r], Tr)
            lse_t = None
        else:
            t = scaled_logits(Ht[r], Wt, Tr)
            lse_t = logsumexp_rows(t)
            l = kl_full_rows(s, lse_s, t, lse_t)
            gr = grad_full_rows(s, lse_s, t, lse_t, Tr)
            if beta > 0:
                l = (1 - beta) * l + beta * kl_reverse_rows(s, lse_s, t, lse_t)
                gr = (1 - beta) * gr + beta * grad_reverse_rows(s, lse_s, t, lse_t, Tr)
        k = keep[r]
        l = np.where(k, l, 0.0)
        dS = np.where(k[:, None], coef * gr, 0.0)
        return l, lse_s, lse_t, dS

    out = {"n_valid": n_valid}
    sel = np.arange(N) if rows is None else _i64(rows)
    vr = np.arange(V) if vocab_rows is None else _i64(vocab_rows)
    row_loss = np.zeros(len(sel))
    lse_s = np.zeros(len(sel))
    lse_t = np.zeros(len(sel)) if mode == HIDDEN else None
    dH = np.zeros((len(sel), d)) if want_dH else None
    dW = np.zeros((len(vr), d)) if want_dW else None
    # dW sums over every token row; when only some rows are evaluated it needs
    # its own pass over all rows.
    dW_in_main = want_dW and rows is None
    for b in range(0, len(sel), block):
        r = sel[b:b + block]
        l, ls, lt, dS = block_terms(r)
        row_loss[b:b + block] = l
        lse_s[b:b + block] = ls
        if lt is not None:
            lse_t[b:b + block] = lt
        if want_dH:
            dH[b:b + block] = dS @ W
        if dW_in_main:
            dW += dS[:, vr].T @ H[r]
    if want_dW and not dW_in_main:
        for b in range(0, N, block):
            r = np.arange(b, min(N, b + block))
            _, _, _, dS = block_terms(r)
            dW += dS[:, vr].T @ H[r]
    out.update(row_loss=row_loss, lse_s=lse_s, lse_t=lse_t, dH=dH, dW=dW)
    if rows is None:
        out["loss"] = float(np.sum(row_loss)) / norm if norm > 0 else 0.0
    return out


def dense_reconstruction_loss(H, W, *, T, topk_idx, topk_logit, teacher_lse=None,
                              mask=None):
    """The dense-reconstruction offline variant of §3 "Offline
    implementations", kept as a second formulation for cross-checks: scatter
    the cached teacher probabilities into a dense [N, V] teacher tensor and
    sum q * (log q - log_softmax(s~)) over the whole vocabulary."""
    H = _f64(H)
    W = _f64(W)
    N = H.shape[0]
    V = W.shape[0]
    idx, q, valid = teacher_support_probs(topk_idx, topk_logit, T, teacher_lse, V)
    dense_q = np.zeros((N, V))
    for n in range(N):
        dense_q[n, idx[n][valid[n]]] = q[n][valid[n]]
    s = scaled_logits(H, W, T)
    log_ps = s - logsumexp_rows(s)[:, None]
    qlogq = np.where(dense_q > 0, dense_q * np.log(np.where(dense_q > 0, dense_q, 1.0)), 0.0)
    l = np.sum(qlogq - dense_q * log_ps, axis=1)
    keep = np.ones(N, dtype=bool) if mask is None else (_i64(mask) != 0)
    nv = int(np.sum(keep))
    return float(np.sum(np.where(keep, l, 0.0)) / nv) if nv else 0.0
