"""Double-buffered host-to-device staging around the fused call.

Three different batches stream from pinned host memory through `HostStager`
while the loss runs; every step must give exactly (bitwise: the kernels are
deterministic) what a direct call on the same batch gives, and the step-0
result must also match the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import _lib as L
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl
from chunked_kl_loss_tma_b200.staging import HostStager

pytestmark = pytest.mark.gpu

NAMES = ("H", "mask", "topk_idx", "topk_logit", "teacher_lse")


def _batch(seed, N=520, d=136, V=3001, K=16):
    w = wl.make_topk("staged", N=N, d=d, V=V, K=K, d_t=64, T=1.5, dtype=torch.bfloat16,
                     w_std=0.05, tw_std=0.1, seed=seed)
    m = torch.ones(N, dtype=torch.uint8)
    m[seed::11] = 0
    w.mask = m
    return w


def test_staged_steps_equal_direct_calls():
    batches = [_batch(s) for s in (21, 22, 23)]
    W = batches[0].W.cuda()          # one resident head for all steps
    for b in batches:
        b.W = batches[0].W
    host = [{k: getattr(b, k).pin_memory() for k in NAMES} for b in batches]
    dev = torch.device("cuda", 0)
    stager = HostStager(host[0], dev, depth=2)
    probs = []
    for s in range(2):
        bf = stager.bufs[s]
        probs.append(ops.make_problem(bf["H"], W, T=1.5, mask=bf["mask"],
                                      topk_idx=bf["topk_idx"], topk_logit=bf["topk_logit"],
                                      teacher_lse=bf["teacher_lse"], chunk_tokens=256))
    ws = ops.alloc_workspace(probs[0][0], L.KL_ENTRY_FWD_BWD, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    dH = torch.empty((batches[0].N, W.shape[1]), dtype=W.dtype, device=dev)
    dW = torch.empty(W.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    outs = []
    slot = stager.put(host[0])
    for i in range(len(host)):
        stager.acquire(slot, stream)
        nxt = stager.put(host[i + 1]) if i + 1 < len(host) else None
        L.check(L.kl_fwd_bwd(probs[slot][0], ws.data_ptr(), ws.numel(), 1.0, loss.data_ptr(),
                             None, dH.data_ptr(), dW.data_ptr(), 0, stream.cuda_stream),
                "kl_fwd_bwd")
        stager.release(slot, stream)
        outs.append((loss.clone(), dH.clone(), dW.clone()))
        slot = nxt
    torch.cuda.synchronize()
    assert ops.status(ws) == 0
    assert stager.bytes_per_step == sum(t.numel() * t.element_size() for t in host[0].values())

    for b, (l_s, dH_s, dW_s) in zip(batches, outs):
        bd = b.to("cuda")
        ref = ops.kl_fwd_bwd(bd.H, W, T=1.5, mask=bd.mask, topk_idx=bd.topk_idx,
                             topk_logit=bd.topk_logit, teacher_lse=bd.teacher_lse,
                             chunk_tokens=256)
        assert torch.equal(l_s, ref["loss"])
        assert torch.equal(dH_s, ref["dH"])
        assert torch.equal(dW_s, ref["dW"])

    b = batches[0]
    o = oracle.kl_loss(b.H, b.W, T=1.5, mask=b.mask, mode="topk", topk_idx=b.topk_idx,
                       topk_logit=b.topk_logit, teacher_lse=b.teacher_lse)
    assert abs(float(outs[0][0]) - o["loss"]) <= 1e-3 * abs(o["loss"])
    err = np.max(np.abs(outs[0][1].double().cpu().numpy() - o["dH"]))
    assert err <= 2e-2 * np.max(np.abs(o["dH"]))


def test_stager_rejects_mismatched_inputs():
    H = torch.zeros(4, 8, dtype=torch.bfloat16)
    st = HostStager({"H": H}, "cuda:0")
    with pytest.raises(KeyError):
        st.put({"X": H})
    with pytest.raises(ValueError):
        st.put({"H": torch.zeros(4, 9, dtype=torch.bfloat16)})
    with pytest.raises(ValueError):
        st.put({"H": H.cuda()})
