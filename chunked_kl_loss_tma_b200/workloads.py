"""Seeded synthetic inputs for the distillation-loss workloads.

This module only draws random inputs and builds the teacher cache the loss
reads; it holds none of the loss's own arithmetic.  The CUDA path (through the
C-ABI) and the fp64 oracle both receive exactly the arrays produced here.

The teacher top-K cache stands in for the cache an inference server writes
once ("Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and a
Fused Chunked KL Loss", §3 "Offline distillation" and App. A): teacher logits
t = Ht . Wt^T of a separate random teacher head on separate random hidden
states, its K largest entries (int32 index + fp32 logit, in descending order)
and the teacher's full-vocabulary log-sum-exp of t/T, with which the loss uses
the cached entries' probabilities without renormalising them over the K.

Workloads (sizes and distributions of the benchmark configurations):
  tiny          N=64, d=64, V=1000, fp32 H~N(0,1), W~N(0,0.05^2); K=8 cache from a
                teacher head d_t=64 (same distributions); T=1; no mask; seed 0.
  offline_topk  N=4096, d=3072, V=128256, bf16 H~N(0,1), W~N(0,0.02^2); K=64 cache
                from a bf16 teacher head N(0,0.02^2), d_t=4096, Ht~N(0,1); T=1.
  full_vocab    N=8192, d=3072, d_t=4096, V=128256, bf16 hiddens N(0,1), both heads
                N(0,0.02^2); teacher logits recomputed by the loss; T=2.
  packed_long   N=32768 packed documents with lengths ~ U[512, 4096]; exactly
                round(0.05 N) positions masked out; otherwise as offline_topk.
  scaling       offline_topk at N in {4096, 16384, 65536, 262144}.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

TOPK = "topk"
HIDDEN = "hidden"


@dataclass
class Workload:
    name: str
    N: int
    d: int
    V: int
    T: "float | torch.Tensor"                    # scalar, or float32 [N] per token
    mode: str
    dtype: torch.dtype
    H: torch.Tensor
    W: torch.Tensor
    mask: Optional[torch.Tensor] = None          # uint8 [N], 1 keep / 0 ignore
    K: int = 0
    topk_idx: Optional[torch.Tensor] = None      # int32 [N, K]
    topk_logit: Optional[torch.Tensor] = None    # fp32 [N, K]
    teacher_lse: Optional[torch.Tensor] = None   # fp32 [N]
    d_t: int = 0
    Ht: Optional[torch.Tensor] = None            # [N, d_t] (hidden mode)
    Wt: Optional[torch.Tensor] = None            # [V, d_t] (hidden mode)
    meta: dict = field(default_factory=dict)

    def to(self, device):
        kw = {}
        for k in ("H", "W", "mask", "topk_idx", "topk_logit", "teacher_lse", "Ht", "Wt", "T"):
            v = getattr(self, k)
            kw[k] = v.to(device) if isinstance(v, torch.Tensor) else v
        return Workload(**{**self.__dict__, **kw})


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, dtype, g, device):
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def teacher_topk_cache(Ht, Wt, K, T, rows_per_block=2048):
    """Teacher cache for rows of Ht: the K largest logits of Ht . Wt^T (fp32
    products of the stored values, descending), their int32 indices, and the
    full-vocabulary log-sum-exp of logits / T (T a number, or a tensor with one
    temperature per row)."""
    N = Ht.shape[0]
    idx = torch.empty(N, K, dtype=torch.int32, device=Ht.device)
    val = torch.empty(N, K, dtype=torch.float32, device=Ht.device)
    lse = torch.empty(N, dtype=torch.float32, device=Ht.device)
    Wf = Wt.float()
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        for b in range(0, N, rows_per_block):
            t = Ht[b:b + rows_per_block].float() @ Wf.T
            v, i = torch.topk(t, K, dim=1, largest=True, sorted=True)
            idx[b:b + rows_per_block] = i.to(torch.int32)
            val[b:b + rows_per_block] = v
            Tb = T[b:b + rows_per_block].to(t.device).double()[:, None] \
                if isinstance(T, torch.Tensor) else T
            lse[b:b + rows_per_block] = torch.logsumexp(t.double() / Tb, dim=1).float()
            del t
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    return idx, val, lse


def make_topk(name, N, d, V, K, d_t, T, dtype, w_std, tw_std, seed, device="cpu",
              mask=None, partial_mass=True, meta=None):
    """Student H, W and a teacher top-K cache from a separate random teacher.
    T may be a float32 tensor [N] of per-token temperatures."""
    g = _gen(seed, device)
    H = _normal((N, d), 1.0, dtype, g, device)
    W = _normal((V, d), w_std, dtype, g, device)
    Ht = _normal((N, d_t), 1.0, dtype, g, device)
    Wt = _normal((V, d_t), tw_std, dtype, g, device)
    idx, val, lse = teacher_topk_cache(Ht, Wt, K, T)
    del Ht, Wt
    return Workload(name=name, N=N, d=d, V=V, T=T, mode=TOPK, dtype=dtype, H=H, W=W,
                    mask=mask, K=K, topk_idx=idx, topk_logit=val,
                    teacher_lse=lse if partial_mass else None, d_t=d_t,
                    meta=dict(meta or {}, seed=seed, partial_mass=partial_mass))


def make_hidden(name, N, d, d_t, V, T, dtype, w_std, tw_std, seed, device="cpu", mask=None):
    """Student H, W and teacher hidden states + frozen teacher head."""
    g = _gen(seed, device)
    H = _normal((N, d), 1.0, dtype, g, device)
    W = _normal((V, d), w_std, dtype, g, device)
    Ht = _normal((N, d_t), 1.0, dtype, g, device)
    Wt = _normal((V, d_t), tw_std, dtype, g, device)
    return Workload(name=name, N=N, d=d, V=V, T=T, mode=HIDDEN, dtype=dtype, H=H, W=W,
                    mask=mask, d_t=d_t, Ht=Ht, Wt=Wt, meta={"seed": seed})


def packed_mask(N, frac, seed, device="cpu", min_len=512, max_len=4096):
    """Document lengths ~ U[min_len, max_len] packed to N tokens (metadata only:
    the loss is per position) and a mask with exactly round(frac * N) positions
    set to 0, chosen uniformly without replacement."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lens, total = [], 0
    while total < N:
        L = int(torch.randint(min_len, max_len + 1, (1,), generator=g))
        L = min(L, N - total)
        lens.append(L)
        total += L
    n_mask = int(round(frac * N))
    perm = torch.randperm(N, generator=g)[:n_mask]
    mask = torch.ones(N, dtype=torch.uint8)
    mask[perm] = 0
    return mask.to(device), lens


def tiny(device="cpu", seed=0, partial_mass=True):
    return make_topk("tiny", N=64, d=64, V=1000, K=8, d_t=64, T=1.0,
                     dtype=torch.float32, w_std=0.05, tw_std=0.05, seed=seed,
                     device=device, partial_mass=partial_mass)


def offline_topk(device="cpu", N=4096, seed=1, partial_mass=True, d=3072, V=128256,
                 K=64, d_t=4096, T=1.0, dtype=torch.bfloat16):
    return make_topk("offline_topk", N=N, d=d, V=V, K=K, d_t=d_t, T=T, dtype=dtype,
                     w_std=0.02, tw_std=0.02, seed=seed, device=device,
                     partial_mass=partial_mass)


def full_vocab(device="cpu", N=8192, seed=2, d=3072, d_t=4096, V=128256, T=2.0,
               dtype=torch.bfloat16):
    return make_hidden("full_vocab", N=N, d=d, d_t=d_t, V=V, T=T, dtype=dtype,
                       w_std=0.02, tw_std=0.02, seed=seed, device=device)


def packed_long(device="cpu", N=32768, seed=3, partial_mass=True, d=3072, V=128256,
                K=64, d_t=4096, T=1.0):
    mask, lens = packed_mask(N, 0.05, seed, device)
    return make_topk("packed_long", N=N, d=d, V=V, K=K, d_t=d_t, T=T,
                     dtype=torch.bfloat16, w_std=0.02, tw_std=0.02, seed=seed,
                     device=device, mask=mask, partial_mass=partial_mass,
                     meta={"doc_lengths": lens})


def scaling(N, device="cpu", seed=4, partial_mass=True):
    return make_topk(f"scaling_{N}", N=N, d=3072, V=128256, K=64, d_t=4096, T=1.0,
                     dtype=torch.bfloat16, w_std=0.02, tw_std=0.02, seed=seed,
                     device=device, partial_mass=partial_mass)
