"""kl_fwd_noalloc: the forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or hand over a workspace (a plugin host
that passes only its input and output buffers, a runtime with a fixed memory
plan, a path where an allocation would synchronise the device).  For them
kl_fwd_noalloc uses a fixed scratch array in the library's static device
memory.  This test calls it through the C ABI twice in a row, on two different
problems, and checks each result against the workspace-based kl_fwd within
the tolerances the parity tests use; it also checks the size and dtype limits.

The file name makes pytest collect it last, so a failure here does not stop a
`-x` run before the other tests."""

import numpy as np
import pytest
import torch

from chunked_kl_loss_tma_b200 import _lib as L
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _noalloc(w, **extra):
    kw = dict(T=w.T, mask=w.mask, topk_idx=w.topk_idx, topk_logit=w.topk_logit,
              teacher_lse=w.teacher_lse)
    kw.update(extra)
    p, keep = ops.make_problem(w.H, w.W, **kw)
    N = w.H.shape[0]
    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    rl = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.full((), -1, dtype=torch.int32, device="cuda")
    rc = L.kl_fwd_noalloc(p, loss.data_ptr(), lse.data_ptr(), rl.data_ptr(), status.data_ptr(),
                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0, L.kl_status_string(rc)
    torch.cuda.synchronize()
    return loss, lse, rl, int(status.item()), kw


def _compare(w, **extra):
    loss, lse, rl, status, kw = _noalloc(w, **extra)
    ref = ops.kl_fwd(w.H, w.W, **kw)
    assert status == 0
    r = ref["loss"].item()
    assert abs(loss.item() - r) <= 1e-3 * abs(r), (loss.item(), r)
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse_s"].cpu().numpy(), rtol=1e-5,
                               atol=1e-5)
    np.testing.assert_allclose(rl.cpu().numpy(), ref["row_loss"].cpu().numpy(), rtol=5e-3,
                               atol=2e-4)


def test_noalloc_matches_kl_fwd_on_two_calls_in_a_row():
    # Call 1: full vocabulary of the benchmark workload; the fixed scratch holds
    # about 1965 token rows at V=128256, K=64, so 4096 tokens take 3 chunks.
    a = wl.offline_topk(device="cuda", N=4096, seed=31)
    _compare(a)
    # Call 2: a different problem (ragged V, renormalised cache, mask, T != 1,
    # several chunks); the scratch still holds call 1's contents.
    b = wl.make_topk("b", N=300, d=200, V=5003, K=16, d_t=64, T=1.3, dtype=torch.bfloat16,
                     w_std=0.05, tw_std=0.1, seed=32, partial_mass=False)
    b.mask = torch.ones(b.N, dtype=torch.uint8)
    b.mask[::7] = 0
    b = b.to("cuda")
    _compare(b, chunk_tokens=100)


def test_noalloc_rejects_what_it_cannot_hold():
    w = wl.make_topk("c", N=8, d=64, V=300, K=4, d_t=16, T=1.0, dtype=torch.float32,
                     w_std=0.1, tw_std=0.1, seed=33).to("cuda")
    p, keep = ops.make_problem(w.H, w.W, topk_idx=w.topk_idx, topk_logit=w.topk_logit)
    out = torch.empty(8, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = L.kl_fwd_noalloc(p, out.data_ptr(), out.data_ptr(), out.data_ptr(), None, stream)
    assert rc == 3  # KL_ERR_DTYPE: bf16 top-K only
    p.dtype = L.KL_DTYPE_BF16
    p.V = 300_000_000  # one row of tile statistics alone exceeds the fixed scratch
    rc = L.kl_fwd_noalloc(p, out.data_ptr(), out.data_ptr(), out.data_ptr(), None, stream)
    assert rc == 11, L.kl_status_string(rc)  # KL_ERR_TOO_LARGE, nothing launched
