"""Vocabulary-parallel form of the fused loss: the output head split by rows.

Tensor-parallel training splits the output layer's vocabulary rows over ranks;
the loss-kernel benchmark of "Efficient Knowledge Distillation for LLMs:
Offline Top-K Logits and a Fused Chunked KL Loss" (§B, toy loss-kernel
benchmark configuration) reports time and memory of its slowest
tensor-parallel rank.  Rank r holds rows [v_begin, v_end) of W (and of the
teacher head Wt); hidden states, mask, temperature and the teacher side are the
same on every rank.  Of the loss's terms only the row log-partition reduces
over the whole vocabulary (same paper, §3 "Offline distillation"), and it
merges from per-shard values, so one exchange of 8 bytes per row and rank per
token chunk suffices:

    for each chunk k:
        kl_vp_fwd_chunk   logits over the shard, row statistics  (kernels)
        all-gather        the P ranks' statistics, rank order    (NCCL)
      [ kl_vp_mid_chunk   the shard's sums (A, U)                (kernels)
        all-gather        the P ranks' sums                      (NCCL) ]
        kl_vp_bwd_chunk   merge, dS, this rank's dH share, own dW rows (kernels)
        all-reduce        the chunk's fp32 dH shares, async      (NCCL)
    all-reduce the loss shares; kl_cast_f32 turns the summed dH into H's dtype.

The bracketed steps run in the teacher-hidden mode with a reverse-KL weight
only: that gradient needs sum_j p_s,j (s~_j - t~_j) over the whole vocabulary
before dS is written.

The arithmetic is in the library's kernels; this module orders the calls and
the collectives.  `emulate` runs P shards one after another on one device
(the gathers and sums become tensor copies and adds), which is how the form is
checked on a single GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib as L
from . import ops

DEFAULT_CHUNK = 4096


def vocab_shard(V_total: int, world: int, rank: int, align: int = 256):
    """[v_begin, v_end) of `rank`'s shard: contiguous, together covering
    [0, V_total) once, boundaries on multiples of `align` (so every shard but the
    last is made of whole 256-row tiles), sizes differing by at most `align`
    (the spare blocks go to the last ranks, which also hold the short final
    block).  Raises if some rank would get no rows."""
    if world < 1 or not 0 <= rank < world or V_total < 1 or align < 1:
        raise ValueError("bad shard request")
    blocks = -(-V_total // align)
    if blocks < world:
        raise ValueError(f"{V_total} rows in blocks of {align} cannot feed {world} ranks")
    base, extra = divmod(blocks, world)
    first_big = world - extra
    b0 = rank * base + max(0, rank - first_big)
    b1 = b0 + base + (1 if rank >= first_big else 0)
    return min(b0 * align, V_total), min(b1 * align, V_total)


def chunk_rows(N: int, chunk_tokens: int = 0):
    """Row ranges of the library's token chunks (the same split as the C ABI)."""
    C = chunk_tokens if chunk_tokens > 0 else DEFAULT_CHUNK
    C = max(1, min(C, N))
    return [(c0, min(C, N - c0)) for c0 in range(0, N, C)]


class ShardPass:
    """One rank's shard of one fused pass: the problem, its workspace and the
    outputs, with the two per-chunk calls of the C ABI."""

    def __init__(self, H, W_shard, *, v_begin, V_total, dW=None, accumulate_dW=False,
                 want_row_loss=False, want_lse=False, workspace=None, **kw):
        self.p, self.keep = ops.make_problem(H, W_shard, v_begin=v_begin, V_total=V_total, **kw)
        dev = H.device
        self.dtype = H.dtype
        self.ws = workspace if workspace is not None else ops.alloc_workspace(
            self.p, L.KL_ENTRY_FWD_BWD, dev)
        n = L.kl_vp_num_chunks(self.p)
        if n < 0:
            raise ValueError("invalid vocabulary-parallel problem")
        self.chunks = chunk_rows(H.shape[0], kw.get("chunk_tokens", 0))
        if len(self.chunks) != n:  # the library's chunking and this module's must agree
            raise RuntimeError(f"chunk count mismatch: {len(self.chunks)} here, {n} in the library")
        N, d = H.shape
        self.loss = torch.zeros((), dtype=torch.float32, device=dev)
        self.row_loss = torch.empty(N, dtype=torch.float32, device=dev) if want_row_loss else None
        self.lse_s = torch.empty(N, dtype=torch.float32, device=dev) if want_lse else None
        self.dH32 = torch.empty(N, d, dtype=torch.float32, device=dev)
        if dW is None:
            dW = torch.empty(W_shard.shape, dtype=torch.float32, device=dev)
            accumulate_dW = False
        ops._need(dW, "dW", torch.float32, dev)
        if dW.shape != W_shard.shape:
            raise ValueError("dW must have the shard's shape")
        self.dW = dW
        self.accumulate = bool(accumulate_dW)
        C = self.chunks[0][1] if self.chunks else 1
        self._stats = torch.empty(C, 2, dtype=torch.float32, device=dev)
        self.two_exchanges = float(kw.get("reverse_weight", 0.0)) > 0.0
        self._sums = torch.empty(C, 2, dtype=torch.float32, device=dev) \
            if self.two_exchanges else None
        self._stream = torch.cuda.current_stream(dev).cuda_stream

    def fwd_chunk(self, k):
        """Chunk k's logits over the shard; returns its row statistics [rows, 2]."""
        rows = self.chunks[k][1]
        st = self._stats[:rows]
        L.check(L.kl_vp_fwd_chunk(self.p, k, self.ws.data_ptr(), self.ws.numel() * self.ws.element_size(), st.data_ptr(),
                                  self._stream), "kl_vp_fwd_chunk")
        return st

    def mid_chunk(self, k, stats_all, P, rank):
        """Chunk k's sums (A, U) over the shard [rows, 2] (reverse-KL weight > 0)."""
        rows = self.chunks[k][1]
        if stats_all.shape != (P * rows, 2) or not stats_all.is_contiguous():
            raise ValueError("stats_all must be a contiguous [P * rows, 2] tensor")
        out = self._sums[:rows]
        L.check(L.kl_vp_mid_chunk(self.p, k, self.ws.data_ptr(), self.ws.numel() * self.ws.element_size(),
                                  stats_all.data_ptr(), P, rank, out.data_ptr(), self._stream),
                "kl_vp_mid_chunk")
        return out

    def bwd_chunk(self, k, stats_all, P, rank, grad_loss=1.0, sums_all=None):
        """Chunk k's gradients from every rank's statistics [P * rows, 2] (rank order)
        and, with a reverse-KL weight, every rank's sums [P * rows, 2]."""
        rows = self.chunks[k][1]
        for t in (stats_all,) + ((sums_all,) if self.two_exchanges else ()):
            if t is None or t.shape != (P * rows, 2) or not t.is_contiguous():
                raise ValueError("statistics must be contiguous [P * rows, 2] tensors")
        L.check(L.kl_vp_bwd_chunk(self.p, k, self.ws.data_ptr(), self.ws.numel() * self.ws.element_size(),
                                  stats_all.data_ptr(), ops._ptr(sums_all), P, rank, grad_loss,
                                  self.loss.data_ptr(), ops._ptr(self.lse_s),
                                  ops._ptr(self.row_loss), self.dH32.data_ptr(),
                                  self.dW.data_ptr(), self.accumulate, self._stream),
                "kl_vp_bwd_chunk")

    def dH_rows(self, k):
        c0, rows = self.chunks[k]
        return self.dH32[c0:c0 + rows]

    def cast_dH(self, src=None):
        """dH in the inputs' dtype from the (summed) fp32 shares."""
        src = self.dH32 if src is None else src
        out = torch.empty(src.shape, dtype=self.dtype, device=src.device)
        L.check(L.kl_cast_f32(src.data_ptr(), out.data_ptr(), src.numel(),
                              L.KL_DTYPE_BF16 if self.dtype == torch.bfloat16 else L.KL_DTYPE_F32,
                              self._stream), "kl_cast_f32")
        return out

    def empty_pass(self):
        """N = 0: no chunk runs; the loss is 0 and dW gets no contribution."""
        if not self.accumulate:
            self.dW.zero_()


class TorchComm:
    """The pass's collectives over a torch.distributed process group: NCCL on
    device tensors (issued even for a group of one rank, so that a one-GPU run
    takes the same path as a multi-GPU one); with another backend (gloo) device
    tensors go through host copies and the reductions run synchronously; with
    no process group, one rank and no collectives."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.nccl = dist.is_initialized() and dist.get_backend(group) == "nccl"

    def all_gather_rows(self, t):
        """[rows, k] from every rank -> [world * rows, k], rank-major."""
        if self.world == 1 and not self.nccl:
            return t
        if self.nccl:
            out = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                              device=t.device)
            dist.all_gather_into_tensor(out, t.contiguous(), group=self.group)
            return out
        h = t.detach().to("cpu").contiguous()
        out = torch.empty((self.world * h.shape[0],) + tuple(h.shape[1:]), dtype=h.dtype)
        dist.all_gather(list(out.split(h.shape[0])), h, group=self.group)
        return out.to(t.device)

    def all_reduce_sum(self, t, async_op=False):
        """In-place sum over ranks; a handle to wait on when async_op and NCCL."""
        if self.world == 1 and not self.nccl:
            return None
        if self.nccl:
            return dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group, async_op=async_op)
        h = t.detach().to("cpu")
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=self.group)
        t.copy_(h)
        return None


def run_pass(shard, comm, grad_loss=1.0):
    """Drive one pass of `shard` (a ShardPass) with `comm`'s collectives.
    Returns dict(loss, row_loss, lse_s, dH, dW), every value the whole
    problem's (dW: this rank's rows)."""
    pending = []
    if not shard.chunks:
        shard.empty_pass()
    for k in range(len(shard.chunks)):
        st_all = comm.all_gather_rows(shard.fwd_chunk(k))
        sums_all = None
        if shard.two_exchanges:
            sums_all = comm.all_gather_rows(shard.mid_chunk(k, st_all, comm.world, comm.rank))
        shard.bwd_chunk(k, st_all, comm.world, comm.rank, grad_loss, sums_all)
        h = comm.all_reduce_sum(shard.dH_rows(k), async_op=True)
        if h is not None:
            pending.append(h)
    for h in pending:
        h.wait()
    comm.all_reduce_sum(shard.loss)
    if shard.row_loss is not None:
        comm.all_reduce_sum(shard.row_loss)
    return dict(loss=shard.loss, row_loss=shard.row_loss, lse_s=shard.lse_s,
                dH=shard.cast_dH(), dW=shard.dW, workspace=shard.ws)


def vp_kl_fwd_bwd(H, W_shard, *, v_begin, V_total, group=None, grad_loss=1.0, **kw):
    """Fused forward + backward of this rank's vocabulary shard inside a
    torch.distributed group (one rank per GPU).  Keywords as ops.kl_fwd_bwd
    (the cache holds whole-vocabulary ids; Wt is this rank's teacher-head
    shard) plus want_lse.  Returns the whole loss, row_loss and dH (identical
    on every rank) and this shard's dW rows."""
    shard = ShardPass(H, W_shard, v_begin=v_begin, V_total=V_total, **kw)
    return run_pass(shard, TorchComm(group), grad_loss)


def emulate(H, W, P, *, shards=None, grad_loss=1.0, Wt=None, **kw):
    """All P ranks of the vocabulary-parallel pass, one after another on one
    device: each shard keeps its own workspace, the all-gathers are
    concatenations and the all-reduces are sums.  Returns the whole loss,
    row_loss, lse_s, dH and the concatenated dW."""
    V = W.shape[0]
    shards = shards or [vocab_shard(V, P, r) for r in range(P)]
    passes = []
    for v0, v1 in shards:
        extra = dict(kw)
        if Wt is not None:
            extra["Wt"] = Wt[v0:v1]
        passes.append(ShardPass(H, W[v0:v1], v_begin=v0, V_total=V, **extra))
    if not passes[0].chunks:
        for s in passes:
            s.empty_pass()
    for k in range(len(passes[0].chunks)):
        stats = torch.cat([s.fwd_chunk(k) for s in passes])
        sums = None
        if passes[0].two_exchanges:
            sums = torch.cat([s.mid_chunk(k, stats, len(passes), r) for r, s in enumerate(passes)])
        for r, s in enumerate(passes):
            s.bwd_chunk(k, stats, len(passes), r, grad_loss, sums)
    loss = sum(s.loss for s in passes)
    row_loss = (sum(s.row_loss for s in passes) if passes[0].row_loss is not None else None)
    dH32 = passes[0].dH32.clone()
    for s in passes[1:]:
        dH32 += s.dH32
    return dict(loss=loss, row_loss=row_loss, lse_s=passes[0].lse_s,
                dH=passes[0].cast_dH(dH32), dW=torch.cat([s.dW for s in passes]),
                workspaces=[s.ws for s in passes])
