"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances (stated by the loss's accuracy target): loss relative error
<= 1e-3; dH and dW max-abs error <= 2e-2 * max|oracle gradient| for bf16 inputs
with fp32 accumulation (and for fp32 inputs through tf32 tensor cores).
Shapes are chosen to span several 128 x 256 tiles with ragged tails in every
dimension (N, d, V not tile multiples, several token chunks with a short
last one)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import _lib as L
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
GRAD_FRAC = 2e-2


def _oracle(w, **kw):
    args = dict(T=w.T, mask=w.mask, mode=w.mode)
    if w.mode == "topk":
        args.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        args.update(Ht=w.Ht, Wt=w.Wt)
    args.update(kw)
    return oracle.kl_loss(w.H, w.W, **args)


def _kw(w, chunk=0, normalizer=0.0):
    kw = dict(T=w.T, mask=w.mask, chunk_tokens=chunk, normalizer=normalizer)
    if w.mode == "topk":
        kw.update(topk_idx=w.topk_idx, topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    else:
        kw.update(Ht=w.Ht, Wt=w.Wt)
    return kw


def _check_grad(got, ref, name):
    got = got.detach().double().cpu().numpy()
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(got - ref))
    assert err <= GRAD_FRAC * scale, f"{name}: max abs err {err:.3e} > {GRAD_FRAC} * {scale:.3e}"
    return err / scale


def _check_loss(got, ref):
    got = float(got)
    assert abs(got - ref) <= LOSS_RTOL * max(abs(ref), 1e-30), f"loss {got} vs oracle {ref}"


def _small_topk(N=300, d=200, V=5003, K=16, dtype=torch.bfloat16, T=1.3, seed=11,
                partial=True, masked=True):
    w = wl.make_topk("small_topk", N=N, d=d, V=V, K=K, d_t=64, T=T, dtype=dtype,
                     w_std=0.05, tw_std=0.1, seed=seed, partial_mass=partial)
    if masked:
        m = torch.ones(N, dtype=torch.uint8)
        m[::7] = 0
        w.mask = m
    return w.to("cuda")


def _small_hidden(N=200, d=136, d_t=72, V=3001, dtype=torch.bfloat16, T=2.0, seed=12):
    w = wl.make_hidden("small_hidden", N=N, d=d, d_t=d_t, V=V, T=T, dtype=dtype,
                       w_std=0.08, tw_std=0.1, seed=seed)
    m = torch.ones(N, dtype=torch.uint8)
    m[3::5] = 0
    w.mask = m
    return w.to("cuda")


@pytest.mark.parametrize("partial", [True, False])
def test_tiny_fp32_fwd_bwd(partial):
    w = wl.tiny(partial_mass=partial).to("cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=2e-3,
                               atol=1e-5)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    assert ops.status(out["workspace"]) == 0


@pytest.mark.parametrize("partial", [True, False])
@pytest.mark.parametrize("chunk", [128, 0])
def test_bf16_topk_ragged_fwd_bwd(partial, chunk):
    w = _small_topk(partial=partial)
    out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=1.7, want_row_loss=True, **_kw(w, chunk))
    ref = _oracle(w, grad_loss=1.7)
    _check_loss(out["loss"].item(), ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=5e-3,
                               atol=2e-4)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    assert ops.status(out["workspace"]) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_hidden_mode_fwd_bwd(dtype):
    w = _small_hidden(dtype=dtype)
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w, chunk=96))
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=5e-3,
                               atol=2e-4)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("mode", ["topk", "hidden"])
def test_split_fwd_then_bwd(mode):
    w = _small_topk() if mode == "topk" else _small_hidden()
    kw = _kw(w, chunk=128)
    f = ops.kl_fwd(w.H, w.W, **kw)
    ref = _oracle(w, grad_loss=0.6)
    _check_loss(f["loss"].item(), ref["loss"])
    np.testing.assert_allclose(f["lse_s"].cpu().numpy(), ref["lse_s"], rtol=1e-5, atol=1e-5)
    if mode == "hidden":
        np.testing.assert_allclose(f["lse_t"].cpu().numpy(), ref["lse_t"], rtol=1e-5, atol=1e-5)
    g = torch.full((), 0.6, device="cuda")
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"], grad_loss=g, **kw)
    _check_grad(b["dH"], ref["dH"], "dH")
    _check_grad(b["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("mode", ["topk", "hidden"])
@pytest.mark.parametrize("chunk", [128, 0])
def test_split_keep_last_chunk(mode, chunk):
    """kl_fwd leaves the last chunk's logits in its workspace and kl_bwd starts
    from them (several chunks with chunk=128, a single one with the default):
    the oracle's loss and gradients, and the recompute-everything backward."""
    w = _small_topk() if mode == "topk" else _small_hidden()
    beta = 0.3 if mode == "hidden" else 0.0
    kw = dict(_kw(w, chunk=chunk), reverse_weight=beta)
    f = ops.kl_fwd(w.H, w.W, keep_last_chunk=True, **kw)
    g = torch.full((), 0.7, device="cuda")
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"], grad_loss=g, workspace=f["workspace"],
                   keep_last_chunk=True, **kw)
    assert ops.status(b["workspace"]) == 0
    ref = _oracle(w, grad_loss=0.7, reverse_weight=beta)
    _check_loss(f["loss"].item(), ref["loss"])
    _check_grad(b["dH"], ref["dH"], "dH")
    _check_grad(b["dW"], ref["dW"], "dW")
    r = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"], grad_loss=g, **kw)
    for k in ("dH", "dW"):
        a, c = b[k].double(), r[k].double()
        assert (a - c).abs().max().item() <= 1e-2 * c.abs().max().item(), k


def test_split_keep_last_chunk_fp32_tiny():
    w = wl.tiny().to("cuda")
    kw = _kw(w, chunk=48)
    f = ops.kl_fwd(w.H, w.W, keep_last_chunk=True, **kw)
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], grad_loss=torch.full((), 1.1, device="cuda"),
                   workspace=f["workspace"], keep_last_chunk=True, **kw)
    ref = _oracle(w, grad_loss=1.1)
    _check_loss(f["loss"].item(), ref["loss"])
    _check_grad(b["dH"], ref["dH"], "dH")
    _check_grad(b["dW"], ref["dW"], "dW")


def test_split_fwd_then_bwd_fp32_tiny():
    w = wl.tiny().to("cuda")
    w.mask = torch.ones(w.N, dtype=torch.uint8, device="cuda")
    w.mask[5::11] = 0
    kw = _kw(w, chunk=48)
    f = ops.kl_fwd(w.H, w.W, **kw)
    ref = _oracle(w, grad_loss=1.3)
    _check_loss(f["loss"].item(), ref["loss"])
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], grad_loss=torch.full((), 1.3, device="cuda"), **kw)
    _check_grad(b["dH"], ref["dH"], "dH")
    _check_grad(b["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("partial", [True, False])
@pytest.mark.parametrize("chunk", [128, 0])
def test_fused_dlogits_path(partial, chunk):
    """fuse_dlogits: the logits pass stores exponentials, the cached entries'
    corrections are folded into them, and dH forms dS in shared memory and
    stores it for dW -- against the oracle, with a mask, several chunks and a
    ragged tail in every dimension, and against the separate dlogits pass."""
    w = _small_topk(partial=partial)
    out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=1.7, want_row_loss=True, fuse_dlogits=True,
                         **_kw(w, chunk))
    assert ops.status(out["workspace"]) == 0
    ref = _oracle(w, grad_loss=1.7)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    plain = ops.kl_fwd_bwd(w.H, w.W, grad_loss=1.7, want_row_loss=True, **_kw(w, chunk))
    assert torch.equal(out["row_loss"], plain["row_loss"])
    for k in ("dH", "dW"):  # differently rounded dS: the gradient tolerance
        a, c = out[k].double(), plain[k].double()
        assert (a - c).abs().max().item() <= GRAD_FRAC * c.abs().max().item(), k


@pytest.mark.parametrize("case", ["K_equals_V", "per_token_T", "accumulate"])
def test_fused_dlogits_edge_cases(case):
    if case == "K_equals_V":
        w = wl.make_topk("kvx", N=96, d=64, V=320, K=320, d_t=32, T=1.0, dtype=torch.bfloat16,
                         w_std=0.1, tw_std=0.2, seed=23).to("cuda")
        kw = _kw(w)
    elif case == "per_token_T":
        Tr = _per_token_T(300, 29)
        w = wl.make_topk("pttx", N=300, d=200, V=5003, K=16, d_t=64, T=Tr, dtype=torch.bfloat16,
                         w_std=0.05, tw_std=0.1, seed=29).to("cuda")
        kw = _kw(w, chunk=128)
    else:
        w = _small_topk(seed=21)
        kw = _kw(w, chunk=64)
    base = torch.randn(w.W.shape, device="cuda", dtype=torch.float32)
    acc = case == "accumulate"
    out = ops.kl_fwd_bwd(w.H, w.W, dW=base.clone() if acc else None, accumulate_dW=acc,
                         fuse_dlogits=True, **kw)
    assert ops.status(out["workspace"]) == 0
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"] - base if acc else out["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("mode,keep,chunk", [("topk", True, 0), ("topk", False, 64),
                                             ("topk", True, 64), ("hidden", True, 64),
                                             ("hidden", False, 64)])
def test_autograd_function_matches_oracle(mode, keep, chunk):
    """fused_kl_loss through autograd: kl_fwd then kl_bwd, with the last chunk's
    logits kept between them or every chunk recomputed."""
    w = _small_topk(N=160, V=2100, masked=False) if mode == "topk" else \
        _small_hidden(N=160, V=2100, seed=33)
    H = w.H.clone().requires_grad_(True)
    W = w.W.clone().requires_grad_(True)
    kw = _kw(w, chunk=chunk)
    loss = ops.fused_kl_loss(H, W, keep_last_chunk=keep, **kw)
    (2.0 * loss).backward()
    ref = _oracle(w, grad_loss=2.0)
    _check_loss(loss.item(), ref["loss"])
    _check_grad(H.grad, ref["dH"], "dH")
    _check_grad(W.grad.float(), ref["dW"], "dW")


def test_accumulate_dW_and_chunk_invariance():
    w = _small_topk(seed=21)
    kw = _kw(w, chunk=64)
    base = torch.randn(w.W.shape, device="cuda", dtype=torch.float32)
    dW = base.clone()
    out = ops.kl_fwd_bwd(w.H, w.W, dW=dW, accumulate_dW=True, **kw)
    ref = _oracle(w)
    _check_grad(out["dW"] - base, ref["dW"], "accumulated dW")
    other = ops.kl_fwd_bwd(w.H, w.W, **_kw(w, chunk=1000))
    assert abs(out["loss"].item() - other["loss"].item()) <= 1e-5 * abs(other["loss"].item())
    _check_grad(other["dH"], out["dH"].double().cpu().numpy(), "dH across chunk sizes")


def test_normalizer_override():
    w = _small_topk(seed=22)
    out = ops.kl_fwd_bwd(w.H, w.W, **_kw(w, normalizer=1000.0))
    ref = _oracle(w, normalizer=1000.0)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dW"], ref["dW"], "dW")


def test_topk_K_equals_V_matches_full_kl():
    V, N = 320, 96
    w = wl.make_topk("kv", N=N, d=64, V=V, K=V, d_t=32, T=1.0, dtype=torch.bfloat16,
                     w_std=0.1, tw_std=0.2, seed=23).to("cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, **_kw(w))
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


def test_empty_slots_and_all_masked_rows():
    w = _small_topk(seed=24, masked=False)
    idx = w.topk_idx.clone()
    idx[:, -3:] = -1
    idx[5, :] = -1  # a row with no cached entry contributes 0
    w.topk_idx = idx
    out = ops.kl_fwd_bwd(w.H, w.W, **_kw(w))
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dW"], ref["dW"], "dW")
    w.mask = torch.zeros(w.N, dtype=torch.uint8, device="cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, **_kw(w))
    assert out["loss"].item() == 0.0
    assert out["dH"].abs().max().item() == 0.0 and out["dW"].abs().max().item() == 0.0


def test_empty_problem():
    H = torch.empty(0, 64, device="cuda", dtype=torch.bfloat16)
    W = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    idx = torch.empty(0, 4, dtype=torch.int32, device="cuda")
    val = torch.empty(0, 4, dtype=torch.float32, device="cuda")
    out = ops.kl_fwd_bwd(H, W, topk_idx=idx, topk_logit=val)
    assert out["loss"].item() == 0.0 and out["dW"].abs().max().item() == 0.0


def test_bad_cache_index_sets_device_status():
    w = _small_topk(seed=25)
    idx = w.topk_idx.clone()
    idx[7, 2] = w.V + 5
    out = ops.kl_fwd_bwd(w.H, w.W, **dict(_kw(w), topk_idx=idx))
    assert ops.status(out["workspace"]) == 7  # KL_ERR_INDEX
    idx = w.topk_idx.clone()
    idx[9, 1] = idx[9, 0]
    out = ops.kl_fwd_bwd(w.H, w.W, **dict(_kw(w), topk_idx=idx))
    assert ops.status(out["workspace"]) == 7
    ok = ops.kl_fwd_bwd(w.H, w.W, **_kw(w))  # status resets on the next call
    assert ops.status(ok["workspace"]) == 0


def test_launch_counter_and_profile():
    w = _small_topk(seed=26)
    before = L.kl_launch_count()
    L.kl_profile_begin()
    ops.kl_fwd_bwd(w.H, w.W, **_kw(w, chunk=128))
    prof = L.kl_profile_end()
    names = {p["name"] for p in prof}
    assert {"gemm_logits_stats", "gemm_dH", "gemm_dW", "dlogits_topk"} <= names
    assert L.kl_launch_count() - before == sum(p["launches"] for p in prof)
    assert all(p["total_ms"] > 0 for p in prof)
    L.kl_profile_begin()
    ops.kl_fwd_bwd(w.H, w.W, fuse_dlogits=True, **_kw(w, chunk=128))
    names = {p["name"] for p in L.kl_profile_end()}
    assert {"gemm_logits_stats", "xf_patch", "xf_scales", "gemm_dH", "gemm_dW"} <= names
    assert "dlogits_topk" not in names
    # teacher-hidden mode: the teacher pass, then the student pass, per chunk
    h = _small_hidden(seed=26)
    L.kl_profile_begin()
    ops.kl_fwd_bwd(h.H, h.W, **_kw(h, chunk=128))
    prof = {p["name"]: p for p in L.kl_profile_end()}
    assert {"gemm_teacher_logits", "gemm_logits_stats", "hidden_sums", "dlogits_full",
            "gemm_dH", "gemm_dW"} <= set(prof)
    chunks = -(-h.N // 128)
    assert prof["gemm_teacher_logits"]["launches"] == prof["gemm_logits_stats"]["launches"] == chunks


def test_binding_rejects_wrong_shapes():
    """The C ABI sees bare pointers, so the binding checks every size the
    kernels rely on and raises before anything is launched."""
    w = _small_topk(seed=28)
    kw = _kw(w)
    N, V = w.N, w.V
    bad = [
        dict(kw, mask=torch.ones(N - 1, dtype=torch.uint8, device="cuda")),
        dict(kw, teacher_lse=torch.zeros(N + 1, device="cuda")),
    ]
    for k in bad:
        with pytest.raises(ValueError):
            ops.kl_fwd_bwd(w.H, w.W, **k)
    with pytest.raises(ValueError):
        ops.kl_fwd_bwd(w.H, w.W, dW=torch.zeros(V - 1, w.d, device="cuda"), **kw)
    f = ops.kl_fwd(w.H, w.W, **kw)
    with pytest.raises(ValueError):
        ops.kl_bwd(w.H, w.W, f["lse_s"][:-1], **kw)
    with pytest.raises(ValueError):
        ops.kl_bwd(w.H, w.W, f["lse_s"], dW=torch.zeros(w.d, V, device="cuda"), **kw)
    h = _small_hidden(seed=29)
    fh = ops.kl_fwd(h.H, h.W, **_kw(h))
    with pytest.raises(ValueError):
        ops.kl_bwd(h.H, h.W, fh["lse_s"], None, **_kw(h))  # lse_t missing
    # a workspace of another element type is measured in bytes
    ws = torch.empty((ops.workspace_bytes(ops.make_problem(w.H, w.W, **kw)[0], 2) + 3) // 4,
                     dtype=torch.float32, device="cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, workspace=ws, **kw)
    assert ops.status(ws) == 0
    ref = ops.kl_fwd_bwd(w.H, w.W, **kw)
    assert torch.equal(out["dW"], ref["dW"])


def test_two_streams_concurrently():
    """Two problems (one per teacher mode) enqueued at once on two streams, each
    with its own workspace: the library keeps no device state outside the
    workspace, so each result equals the same call run alone, bit for bit."""
    a = _small_topk(seed=30)
    b = _small_hidden(seed=31)
    ka, kb = _kw(a, chunk=128), _kw(b, chunk=96)
    ref_a = ops.kl_fwd_bwd(a.H, a.W, **ka)
    ref_b = ops.kl_fwd_bwd(b.H, b.W, **kb)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            oa = ops.kl_fwd_bwd(a.H, a.W, **ka)
        with torch.cuda.stream(s2):
            ob = ops.kl_fwd_bwd(b.H, b.W, **kb)
        outs.append((oa, ob))
    torch.cuda.synchronize()
    for oa, ob in outs:
        assert ops.status(oa["workspace"]) == 0 and ops.status(ob["workspace"]) == 0
        for k in ("loss", "dH", "dW"):
            assert torch.equal(oa[k], ref_a[k]), ("topk", k)
            assert torch.equal(ob[k], ref_b[k]), ("hidden", k)


def test_bitwise_deterministic_across_calls():
    """Every reduction has a fixed order (per-row statistics, split-V merge,
    split-K parts, per-chunk dW add-reductions issued in chunk order), so two
    calls on the same inputs agree bit for bit."""
    w = _small_topk(seed=27)
    kw = _kw(w, chunk=96)
    a = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    b = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    for k in ("loss", "row_loss", "dH", "dW"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("beta", [1.0, 0.35])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_reverse_and_mixed_kl_fused_and_split(beta, dtype):
    w = _small_hidden(dtype=dtype, seed=28)
    kw = dict(_kw(w, chunk=96), reverse_weight=beta)
    ref = _oracle(w, reverse_weight=beta, grad_loss=1.4)
    out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=1.4, want_row_loss=True, **kw)
    _check_loss(out["loss"].item(), ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=5e-3,
                               atol=2e-4)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    f = ops.kl_fwd(w.H, w.W, **kw)
    _check_loss(f["loss"].item(), ref["loss"])
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"],
                   grad_loss=torch.full((), 1.4, device="cuda"), **kw)
    _check_grad(b["dH"], ref["dH"], "dH (split)")
    _check_grad(b["dW"], ref["dW"], "dW (split)")


def _per_token_T(N, seed):
    g = torch.Generator().manual_seed(seed)
    return (0.5 + 2.0 * torch.rand(N, generator=g)).float()


@pytest.mark.parametrize("partial", [True, False])
def test_per_token_temperature_topk_fused_and_split(partial):
    Tr = _per_token_T(300, 29)
    w = wl.make_topk("ptt", N=300, d=200, V=5003, K=16, d_t=64, T=Tr, dtype=torch.bfloat16,
                     w_std=0.05, tw_std=0.1, seed=29, partial_mass=partial).to("cuda")
    w.mask = torch.ones(300, dtype=torch.uint8, device="cuda")
    w.mask[::6] = 0
    kw = _kw(w, chunk=128)
    ref = _oracle(w, grad_loss=0.8)
    out = ops.kl_fwd_bwd(w.H, w.W, grad_loss=0.8, want_row_loss=True, **kw)
    assert ops.status(out["workspace"]) == 0
    _check_loss(out["loss"].item(), ref["loss"])
    np.testing.assert_allclose(out["row_loss"].cpu().numpy(), ref["row_loss"], rtol=5e-3,
                               atol=2e-4)
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    f = ops.kl_fwd(w.H, w.W, **kw)
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], grad_loss=torch.full((), 0.8, device="cuda"), **kw)
    _check_loss(f["loss"].item(), ref["loss"])
    _check_grad(b["dH"], ref["dH"], "dH (split)")
    _check_grad(b["dW"], ref["dW"], "dW (split)")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_per_token_temperature_hidden_mixed(dtype):
    w = _small_hidden(dtype=dtype, seed=30)
    w.T = _per_token_T(w.N, 30).to("cuda")
    kw = dict(_kw(w, chunk=96), reverse_weight=0.25)
    ref = _oracle(w, reverse_weight=0.25)
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


def test_non_positive_per_token_temperature_sets_status():
    w = _small_topk(seed=31)
    Tr = torch.ones(w.N, device="cuda")
    Tr[17] = 0.0
    out = ops.kl_fwd_bwd(w.H, w.W, **dict(_kw(w), T=Tr))
    assert ops.status(out["workspace"]) == 10  # KL_ERR_ARG


def test_max_cache_size_K1024():
    w = wl.make_topk("k1024", N=130, d=64, V=2000, K=1024, d_t=32, T=1.2,
                     dtype=torch.bfloat16, w_std=0.1, tw_std=0.2, seed=32).to("cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, **_kw(w, chunk=64))
    assert ops.status(out["workspace"]) == 0
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("mode,d,d_t", [("topk", 8192, 64), ("hidden", 8192, 1024),
                                         ("hidden", 512, 8192)])
def test_wide_heads(mode, d, d_t):
    """Hidden widths well above the bench's 3072 (128 K-blocks per logits tile,
    8192-wide dH rows and dW columns), through the fused call and the split pair
    with the last chunk kept, with a ragged last chunk."""
    if mode == "topk":
        w = wl.make_topk("wide", N=300, d=d, V=1500, K=32, d_t=d_t, T=1.5,
                         dtype=torch.bfloat16, w_std=0.02, tw_std=0.05, seed=41).to("cuda")
    else:
        w = wl.make_hidden("wideh", N=300, d=d, d_t=d_t, V=1500, T=1.5, dtype=torch.bfloat16,
                           w_std=0.02, tw_std=0.02, seed=42).to("cuda")
    ref = _oracle(w)
    kw = _kw(w, chunk=128)
    out = ops.kl_fwd_bwd(w.H, w.W, **kw)
    assert ops.status(out["workspace"]) == 0
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")
    f = ops.kl_fwd(w.H, w.W, keep_last_chunk=True, **kw)
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], f["lse_t"], workspace=f["workspace"],
                   keep_last_chunk=True, **kw)
    assert ops.status(f["workspace"]) == 0
    _check_loss(f["loss"].item(), ref["loss"])
    _check_grad(b["dH"], ref["dH"], "dH (split)")
    _check_grad(b["dW"], ref["dW"], "dW (split)")


@pytest.mark.parametrize("mode", ["topk", "hidden"])
def test_vocabulary_262144(mode):
    """A 2^18-entry vocabulary (1024 tiles of 256 columns per row, twice the
    bench's): the split-V merge over all tiles, cache ids up to 262143 and the
    gradients, fused call with a ragged chunk."""
    V = 262144
    if mode == "topk":
        w = wl.make_topk("v256k", N=200, d=128, V=V, K=64, d_t=64, T=1.2, dtype=torch.bfloat16,
                         w_std=0.1, tw_std=0.2, seed=43).to("cuda")
    else:
        w = wl.make_hidden("v256kh", N=200, d=128, d_t=96, V=V, T=1.7, dtype=torch.bfloat16,
                           w_std=0.1, tw_std=0.1, seed=44).to("cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w, chunk=128))
    assert ops.status(out["workspace"]) == 0
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


@pytest.mark.parametrize("mode", ["topk", "hidden"])
def test_vocabulary_smaller_than_one_tile(mode):
    if mode == "topk":
        w = wl.make_topk("v40", N=70, d=32, V=40, K=40, d_t=16, T=0.9, dtype=torch.bfloat16,
                         w_std=0.2, tw_std=0.3, seed=33).to("cuda")
    else:
        w = wl.make_hidden("v40h", N=70, d=32, d_t=16, V=40, T=0.9, dtype=torch.bfloat16,
                           w_std=0.2, tw_std=0.3, seed=33).to("cuda")
    out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **_kw(w))
    ref = _oracle(w)
    _check_loss(out["loss"].item(), ref["loss"])
    _check_grad(out["dH"], ref["dH"], "dH")
    _check_grad(out["dW"], ref["dW"], "dW")


def test_split_backward_accumulates_into_dW():
    w = _small_topk(seed=34)
    kw = _kw(w, chunk=128)
    f = ops.kl_fwd(w.H, w.W, **kw)
    base = torch.randn(w.W.shape, device="cuda", dtype=torch.float32)
    b = ops.kl_bwd(w.H, w.W, f["lse_s"], dW=base.clone(), accumulate_dW=True, **kw)
    ref = _oracle(w)
    _check_grad(b["dW"] - base, ref["dW"], "accumulated dW (split)")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N,d,V,K", [(1, 8, 1, 1), (3, 8, 7, 2), (5, 16, 9, 9), (2, 8, 300, 1)])
def test_smallest_shapes(dtype, N, d, V, K):
    """One-row, one-class and sub-vector vocabularies (V < 8 pads the logit
    rows), the narrowest width d = 8 and a single cached entry, both teacher
    modes.  With V = 1 both distributions are a point mass: loss 0 up to
    rounding, so the loss is held to 1e-3 relative plus an absolute 1e-6 that
    only matters when the oracle's loss is itself zero."""
    w = wl.make_topk("tiny_shapes", N=N, d=d, V=V, K=K, d_t=8, T=1.1, dtype=dtype,
                     w_std=0.3, tw_std=0.3, seed=50 + V).to("cuda")
    for partial in (True, False):
        kw = _kw(w)
        if not partial:
            kw["teacher_lse"] = None
        out = ops.kl_fwd_bwd(w.H, w.W, want_row_loss=True, **kw)
        assert ops.status(out["workspace"]) == 0
        ref = _oracle(w, teacher_lse=kw["teacher_lse"])
        assert abs(out["loss"].item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]) + 1e-6
        for k in ("dH", "dW"):
            got = out[k].double().cpu().numpy()
            assert np.max(np.abs(got - ref[k])) <= GRAD_FRAC * np.max(np.abs(ref[k])) + 1e-6, k
    h = wl.make_hidden("tiny_shapes_h", N=N, d=d, d_t=8, V=V, T=1.1, dtype=dtype, w_std=0.3,
                       tw_std=0.3, seed=60 + V).to("cuda")
    out = ops.kl_fwd_bwd(h.H, h.W, want_row_loss=True, **_kw(h))
    ref = _oracle(h)
    assert abs(out["loss"].item() - ref["loss"]) <= 1e-3 * abs(ref["loss"]) + 1e-6
    for k in ("dH", "dW"):
        got = out[k].double().cpu().numpy()
        assert np.max(np.abs(got - ref[k])) <= GRAD_FRAC * np.max(np.abs(ref[k])) + 1e-6, k
