"""Host logic of the vocabulary-parallel pass on CPU: shard boundaries, and
`run_pass` driving two and three gloo ranks (top-K mode with one exchange per chunk, and
teacher-hidden mode with a reverse-KL weight and two exchanges).

Each rank's per-chunk compute here is a small numpy stand-in written from the
decomposition the library uses (per-shard log-sum-exp and cross term, merged
over ranks; dS over the shard's columns; dH shares summed over ranks).  The
pass's result must equal the fp64 oracle's whole-head loss and gradients,
which checks the collectives' order and sums, and the decomposition itself,
without a GPU.  The CUDA kernels of the same steps are checked against the
oracle in test_vocab_parallel_gpu.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunked_kl_loss_tma_b200.vocab_parallel import TorchComm, chunk_rows, run_pass, vocab_shard


def test_vocab_shards_cover_the_head_on_tile_boundaries():
    for V in (256, 257, 5003, 128256):
        for world in (1, 2, 3, 8):
            if -(-V // 256) < world:
                with pytest.raises(ValueError):
                    vocab_shard(V, world, 0)
                continue
            got = [vocab_shard(V, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == V
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            assert all(b > a for a, b in got)
            assert all(a % 256 == 0 for a, _ in got)
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 256
    assert vocab_shard(128256, 8, 7) == (112128, 128256)
    with pytest.raises(ValueError):
        vocab_shard(100, 2, 2)


def test_chunk_rows_match_the_library_split():
    assert chunk_rows(0) == []
    assert chunk_rows(300, 128) == [(0, 128), (128, 128), (256, 44)]
    assert chunk_rows(5000) == [(0, 4096), (4096, 904)]
    assert chunk_rows(7, 4096) == [(0, 7)]


def _lse(x, axis):
    m = np.max(x, axis=axis, keepdims=True)
    return np.squeeze(m, axis) + np.log(np.sum(np.exp(x - m), axis=axis))


class NumpyShard:
    """Stand-in for ShardPass (top-K, partial mass) with numpy arithmetic."""

    def __init__(self, H, W, v0, v1, idx, logit, lse_t, T, mask, chunk):
        self.H, self.Ws, self.v0, self.v1 = H, W[v0:v1], v0, v1
        self.idx, self.T, self.mask = idx, T, mask
        self.q = np.where(idx >= 0, np.exp(logit / T - lse_t[:, None]), 0.0)
        self.n_valid = int(mask.sum())
        N, d = H.shape
        self.chunks = chunk_rows(N, chunk)
        self.loss = torch.zeros((), dtype=torch.float64)
        self.row_loss = torch.zeros(N, dtype=torch.float64)
        self.lse_s = torch.zeros(N, dtype=torch.float64)
        self.dH32 = torch.zeros(N, d, dtype=torch.float64)
        self.dW = torch.zeros(v1 - v0, d, dtype=torch.float64)
        self.two_exchanges = False  # top-K mode: one exchange per chunk
        self.ws = None

    def _local(self, rows):
        """Cached entries of these rows inside the shard: (row, local col, q)."""
        r, k = np.nonzero((self.idx[rows] >= self.v0) & (self.idx[rows] < self.v1))
        return r, self.idx[rows][r, k] - self.v0, self.q[rows][r, k]

    def fwd_chunk(self, k):
        c0, n = self.chunks[k]
        rows = slice(c0, c0 + n)
        self._s = self.H[rows] @ self.Ws.T / self.T
        r, c, q = self._local(rows)
        cross = np.bincount(r, weights=q * self._s[r, c], minlength=n)
        return torch.tensor(np.stack([_lse(self._s, 1), cross], 1))

    def bwd_chunk(self, k, stats_all, P, rank, grad_loss=1.0, sums_all=None):
        c0, n = self.chunks[k]
        rows = slice(c0, c0 + n)
        st = stats_all.numpy().reshape(P, n, 2)
        lse = _lse(st[:, :, 0], 0)
        cross = st[:, :, 1].sum(0)
        q = self.q[rows]
        m = q.sum(1)
        ent = np.sum(np.where(q > 0, q * np.log(np.where(q > 0, q, 1.0)), 0.0), 1)
        keep = self.mask[rows] != 0
        self.lse_s[rows] = torch.tensor(lse)
        self.row_loss[rows] = torch.tensor(np.where(keep & (rank == 0), ent - cross + m * lse, 0))
        coef = np.where(keep, grad_loss / self.n_valid / self.T, 0.0)
        dS = m[:, None] * np.exp(self._s - lse[:, None])
        r, c, qq = self._local(rows)
        np.subtract.at(dS, (r, c), qq)
        dS *= coef[:, None]
        self.dH32[rows] = torch.tensor(dS @ self.Ws)
        self.dW += torch.tensor(dS.T @ self.H[rows])
        if c0 + n == self.H.shape[0]:
            self.loss.fill_(float(self.row_loss.sum()) / self.n_valid)

    def dH_rows(self, k):
        c0, n = self.chunks[k]
        return self.dH32[c0:c0 + n]

    def cast_dH(self):
        return self.dH32.clone()

    def empty_pass(self):
        self.dW.zero_()


def _problem():
    rng = np.random.default_rng(7)  # the same whole problem on every rank
    N, d, V, K, T = 21, 6, 37, 5, 1.3
    H = rng.normal(size=(N, d))
    W = rng.normal(scale=0.6, size=(V, d))
    t = rng.normal(size=(N, V))
    idx = np.argsort(-t, axis=1)[:, :K].astype(np.int64)
    logit = np.take_along_axis(t, idx, 1)
    lse_t = _lse(t / T, 1)
    idx[2, 1:] = -1  # empty slots
    mask = (rng.random(N) > 0.25).astype(np.uint8)
    return H, W, idx, logit, lse_t, T, mask


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
        H, W, idx, logit, lse_t, T, mask = _problem()
        v0, v1 = vocab_shard(W.shape[0], world, rank, align=8)
        shard = NumpyShard(H, W, v0, v1, idx, logit, lse_t, T, mask, chunk=8)
        out = run_pass(shard, TorchComm(), grad_loss=0.9)
        ref = oracle.kl_loss(H, W, T=T, mask=mask, topk_idx=idx, topk_logit=logit,
                             teacher_lse=lse_t, grad_loss=0.9)
        q.put((rank, float(out["loss"]) - ref["loss"],
               float(np.max(np.abs(out["row_loss"].numpy() - ref["row_loss"]))),
               float(np.max(np.abs(out["lse_s"].numpy() - ref["lse_s"]))),
               float(np.max(np.abs(out["dH"].numpy() - ref["dH"]))),
               float(np.max(np.abs(out["dW"].numpy() - ref["dW"][v0:v1]))),
               float(np.max(np.abs(ref["dH"])))))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocabulary_parallel_pass_matches_whole_head_oracle(world):
    """world ranks of gloo, each with its vocabulary shard (3 ranks: uneven shards)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert len(r) == 7, r
    for rank, dloss, drow, dlse, ddH, ddW, scale in res:
        assert scale > 1e-3
        assert abs(dloss) < 1e-12 and drow < 1e-12 and dlse < 1e-12, rank
        assert ddH < 1e-12 and ddW < 1e-12, rank


class NumpyHiddenShard:
    """Stand-in for ShardPass in the teacher-hidden mode with a reverse-KL weight:
    the two exchanges of run_pass (row lse's, then the sums A and U)."""

    def __init__(self, H, W, Ht, Wt, v0, v1, T, mask, beta, chunk):
        self.H, self.Ht, self.Ws, self.Wts = H, Ht, W[v0:v1], Wt[v0:v1]
        self.T, self.mask, self.beta = T, mask, beta
        self.n_valid = int(mask.sum())
        N, d = H.shape
        self.chunks = chunk_rows(N, chunk)
        self.loss = torch.zeros((), dtype=torch.float64)
        self.row_loss = torch.zeros(N, dtype=torch.float64)
        self.lse_s = torch.zeros(N, dtype=torch.float64)
        self.dH32 = torch.zeros(N, d, dtype=torch.float64)
        self.dW = torch.zeros(v1 - v0, d, dtype=torch.float64)
        self.two_exchanges = True
        self.ws = None

    def fwd_chunk(self, k):
        c0, n = self.chunks[k]
        rows = slice(c0, c0 + n)
        self._s = self.H[rows] @ self.Ws.T / self.T
        self._t = self.Ht[rows] @ self.Wts.T / self.T
        return torch.tensor(np.stack([_lse(self._s, 1), _lse(self._t, 1)], 1))

    def _merged(self, stats_all, P, n):
        st = stats_all.numpy().reshape(P, n, 2)
        return _lse(st[:, :, 0], 0), _lse(st[:, :, 1], 0)

    def mid_chunk(self, k, stats_all, P, rank):
        n = self.chunks[k][1]
        ls, lt = self._merged(stats_all, P, n)
        ps = np.exp(self._s - ls[:, None])
        pt = np.exp(self._t - lt[:, None])
        u = self._s - self._t
        return torch.tensor(np.stack([np.sum(-pt * u, 1), np.sum(ps * u, 1)], 1))

    def bwd_chunk(self, k, stats_all, P, rank, grad_loss=1.0, sums_all=None):
        c0, n = self.chunks[k]
        rows = slice(c0, c0 + n)
        ls, lt = self._merged(stats_all, P, n)
        sums = sums_all.numpy().reshape(P, n, 2)
        A, U = sums[rank, :, 0], sums[rank, :, 1]
        ubar = sums[:, :, 1].sum(0)
        b = self.beta
        keep = self.mask[rows] != 0
        dl = (ls - lt) if rank == 0 else 0.0
        self.lse_s[rows] = torch.tensor(ls)
        self.row_loss[rows] = torch.tensor(np.where(keep, (1 - b) * (A + dl) + b * (U - dl), 0))
        ps = np.exp(self._s - ls[:, None])
        pt = np.exp(self._t - lt[:, None])
        u = self._s - self._t
        coef = np.where(keep, grad_loss / self.n_valid / self.T, 0.0)
        dS = coef[:, None] * ((1 - b) * (ps - pt) + b * ps * (u - ubar[:, None]))
        self.dH32[rows] = torch.tensor(dS @ self.Ws)
        self.dW += torch.tensor(dS.T @ self.H[rows])
        if c0 + n == self.H.shape[0]:
            self.loss.fill_(float(self.row_loss.sum()) / self.n_valid)

    def dH_rows(self, k):
        c0, n = self.chunks[k]
        return self.dH32[c0:c0 + n]

    def cast_dH(self):
        return self.dH32.clone()

    def empty_pass(self):
        self.dW.zero_()


def _hidden_worker(rank, world, port, q):
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(11)  # the same whole problem on every rank
        N, d, d_t, V, T, beta = 19, 5, 7, 29, 1.7, 0.4
        H, Ht = rng.normal(size=(N, d)), rng.normal(size=(N, d_t))
        W, Wt = rng.normal(scale=0.5, size=(V, d)), rng.normal(scale=0.5, size=(V, d_t))
        mask = (rng.random(N) > 0.2).astype(np.uint8)
        v0, v1 = vocab_shard(V, world, rank, align=8)
        shard = NumpyHiddenShard(H, W, Ht, Wt, v0, v1, T, mask, beta, chunk=6)
        out = run_pass(shard, TorchComm(), grad_loss=1.3)
        ref = oracle.kl_loss(H, W, T=T, mask=mask, mode="hidden", Ht=Ht, Wt=Wt,
                             reverse_weight=beta, grad_loss=1.3)
        q.put((rank, float(out["loss"]) - ref["loss"],
               float(np.max(np.abs(out["row_loss"].numpy() - ref["row_loss"]))),
               float(np.max(np.abs(out["dH"].numpy() - ref["dH"]))),
               float(np.max(np.abs(out["dW"].numpy() - ref["dW"][v0:v1]))),
               float(np.max(np.abs(ref["dH"])))))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_reverse_kl_pass_with_two_exchanges_matches_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_hidden_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert len(r) == 6, r
        rank, dloss, drow, ddH, ddW, scale = r
        assert scale > 1e-3
        assert abs(dloss) < 1e-12 and drow < 1e-12 and ddH < 1e-12 and ddW < 1e-12, r
