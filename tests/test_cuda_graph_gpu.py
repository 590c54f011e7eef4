"""The C ABI's calls inside a CUDA graph.  Every call is asynchronous on the
caller's stream and reads no device value on the host, so a training loop can
capture it once and replay it with new inputs copied into the captured
tensors.  A replay runs the same kernels in the same order as an eager call, so
the results agree bit for bit.  The status word lives in the workspace, and it
reads 0 after the replays."""
import pytest
import torch

from chunked_kl_loss_tma_b200 import _lib as L
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Warm up on a side stream (first-call attribute setup happens outside the
    capture), then capture fn() into a graph.  Returns (graph, outputs)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


def _equal(a, b):
    return a is None and b is None or torch.equal(a, b)


def test_fused_call_in_a_graph_topk():
    data = [wl.make_topk(f"graph{i}", N=300, d=136, V=3001, K=16, d_t=64, T=1.4,
                         dtype=torch.bfloat16, w_std=0.08, tw_std=0.1, seed=80 + i).to("cuda")
            for i in range(2)]
    m = torch.ones(300, dtype=torch.uint8, device="cuda")
    m[::7] = 0
    # the captured inputs: every replay reads whatever they hold
    H = data[0].H.clone()
    W = data[0].W.clone()
    idx = data[0].topk_idx.clone()
    val = data[0].topk_logit.clone()
    lse = data[0].teacher_lse.clone()
    dW = torch.zeros(W.shape, dtype=torch.float32, device="cuda")
    ws = ops.alloc_workspace(
        ops.make_problem(H, W, T=1.4, topk_idx=idx, topk_logit=val, teacher_lse=lse, mask=m,
                         chunk_tokens=128)[0], L.KL_ENTRY_FWD_BWD, H.device)

    def step():
        return ops.kl_fwd_bwd(H, W, T=1.4, topk_idx=idx, topk_logit=val, teacher_lse=lse,
                              mask=m, chunk_tokens=128, grad_loss=0.9, want_row_loss=True,
                              dW=dW, workspace=ws)

    g, out = _capture(step)
    for w in data + data[:1]:
        for dst, src in ((H, w.H), (W, w.W), (idx, w.topk_idx), (val, w.topk_logit),
                         (lse, w.teacher_lse)):
            dst.copy_(src)
        g.replay()
        got = {k: out[k].clone() for k in ("loss", "row_loss", "dH", "dW")}
        assert ops.status(ws) == 0
        ref = ops.kl_fwd_bwd(w.H, w.W, T=1.4, topk_idx=w.topk_idx, topk_logit=w.topk_logit,
                             teacher_lse=w.teacher_lse, mask=m, chunk_tokens=128,
                             grad_loss=0.9, want_row_loss=True)
        for k in got:
            assert _equal(got[k], ref[k]), k


def test_split_calls_in_a_graph_hidden_keep_last_chunk():
    """kl_fwd then kl_bwd (the autograd pair, the last chunk's logits kept in
    the workspace between them), teacher-hidden with a reverse-KL weight and a
    per-token temperature, captured together in one graph."""
    data = [wl.make_hidden(f"graphh{i}", N=200, d=96, d_t=72, V=2100, T=1.5,
                           dtype=torch.bfloat16, w_std=0.08, tw_std=0.1, seed=90 + i).to("cuda")
            for i in range(2)]
    T_row = torch.linspace(0.8, 2.5, 200, device="cuda")
    H, W = data[0].H.clone(), data[0].W.clone()
    Ht, Wt = data[0].Ht.clone(), data[0].Wt.clone()
    gl = torch.full((), 1.3, device="cuda")
    kw = dict(T=T_row, reverse_weight=0.3, chunk_tokens=64, keep_last_chunk=True)

    def step(H=H, W=W, Ht=Ht, Wt=Wt):
        f = ops.kl_fwd(H, W, Ht=Ht, Wt=Wt, **kw)
        b = ops.kl_bwd(H, W, f["lse_s"], f["lse_t"], grad_loss=gl, Ht=Ht, Wt=Wt,
                       workspace=f["workspace"], **kw)
        return dict(loss=f["loss"], dH=b["dH"], dW=b["dW"], ws=f["workspace"])

    g, out = _capture(step)
    for w in reversed(data):
        for dst, src in ((H, w.H), (W, w.W), (Ht, w.Ht), (Wt, w.Wt)):
            dst.copy_(src)
        g.replay()
        got = {k: out[k].clone() for k in ("loss", "dH", "dW")}
        assert ops.status(out["ws"]) == 0
        ref = step(w.H, w.W, w.Ht, w.Wt)
        for k in got:
            assert _equal(got[k], ref[k]), k
