"""Pins for the fp64 oracle against what the pages and the mathematics fix.

Every pin is independent of the oracle's own code: hand-derived closed forms
(tests/golden/closed_forms.json), a library KL routine (scipy), torch autograd,
central finite differences, K = V equivalence between the top-K and the
full-vocabulary forms, the dense-reconstruction formulation of §3 "Offline
implementations" (Efficient Knowledge Distillation for LLMs: Offline Top-K
Logits and a Fused Chunked KL Loss), and invariants (masking, empty slots,
permutations, temperature scaling, row sampling).  The mutation tests at the
end plant mistakes in the oracle (on the CPU) and check that a pin catches
each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import oracle
from oracle import kl_oracle as ko

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _ev(x):
    if isinstance(x, str):
        return np.array(eval(x, {"math": math}), dtype=np.float64)  # noqa: S307 - fixture expressions
    return None if x is None else np.array(x, dtype=np.float64)


def _rand_case(seed, N=6, d=5, V=13, K=4, d_t=3, mode="topk", partial=True, masked=True,
               T=1.3):
    rng = np.random.default_rng(seed)
    H = rng.normal(size=(N, d))
    W = rng.normal(scale=0.7, size=(V, d))
    Ht = rng.normal(size=(N, d_t))
    Wt = rng.normal(scale=0.9, size=(V, d_t))
    mask = None
    if masked:
        mask = np.ones(N, dtype=np.uint8)
        mask[rng.choice(N, size=max(1, N // 3), replace=False)] = 0
    kw = dict(T=T, mask=mask)
    if mode == "topk":
        t = Ht @ Wt.T
        idx = np.argsort(-t, axis=1)[:, :K].astype(np.int32)
        logit = np.take_along_axis(t, idx, axis=1)
        lse = scipy.special.logsumexp(t / T, axis=1) if partial else None
        kw.update(mode="topk", topk_idx=idx, topk_logit=logit, teacher_lse=lse)
    else:
        kw.update(mode="hidden", Ht=Ht, Wt=Wt)
    return H, W, kw


# ----------------------------------------------------------------------------- golden

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_closed_forms(case):
    kw = dict(T=case["T"], mode=case["mode"], reverse_weight=case.get("reverse_weight", 0.0))
    if case.get("mask") is not None:
        kw["mask"] = np.array(case["mask"], dtype=np.uint8)
    if case["mode"] == "topk":
        kw.update(topk_idx=np.array(case["topk_idx"], dtype=np.int32),
                  topk_logit=_ev(case["topk_logit"]), teacher_lse=_ev(case["teacher_lse"]))
    else:
        kw.update(Ht=_ev(case["Ht"]), Wt=_ev(case["Wt"]))
    out = oracle.kl_loss(_ev(case["H"]), _ev(case["W"]), **kw)
    assert out["loss"] == pytest.approx(float(_ev(case["loss"])), abs=1e-13, rel=1e-12)
    np.testing.assert_allclose(out["dH"], _ev(case["dH"]), atol=1e-13, rtol=1e-12)
    np.testing.assert_allclose(out["dW"], _ev(case["dW"]), atol=1e-13, rtol=1e-12)


# ------------------------------------------------------------------ library routines

def test_full_mode_rows_match_scipy_entropy():
    H, W, kw = _rand_case(1, N=7, d=4, V=17, mode="hidden", masked=False, T=1.7)
    out = oracle.kl_loss(H, W, **kw)
    p_s = scipy.special.softmax(H @ W.T / 1.7, axis=1)
    p_t = scipy.special.softmax(kw["Ht"] @ kw["Wt"].T / 1.7, axis=1)
    for n in range(H.shape[0]):
        assert out["row_loss"][n] == pytest.approx(scipy.stats.entropy(p_t[n], p_s[n]),
                                                   rel=1e-12, abs=1e-14)
    assert out["loss"] == pytest.approx(np.mean(out["row_loss"]), rel=1e-13)
    np.testing.assert_allclose(out["lse_s"], scipy.special.logsumexp(H @ W.T / 1.7, axis=1),
                               rtol=1e-13)


def test_full_mode_matches_torch_kl_div_and_autograd():
    H, W, kw = _rand_case(2, N=8, d=6, V=19, mode="hidden", masked=True, T=0.8)
    out = oracle.kl_loss(H, W, grad_loss=1.0, **kw)
    Ht_ = torch.tensor(H, requires_grad=True)
    Wt_ = torch.tensor(W, requires_grad=True)
    keep = torch.tensor(kw["mask"]).bool()
    log_ps = torch.log_softmax(Ht_ @ Wt_.T / 0.8, dim=1)
    log_pt = torch.log_softmax(torch.tensor(kw["Ht"]) @ torch.tensor(kw["Wt"]).T / 0.8, dim=1)
    rows = torch.nn.functional.kl_div(log_ps, log_pt, reduction="none", log_target=True).sum(1)
    L = rows[keep].mean()
    L.backward()
    assert out["loss"] == pytest.approx(L.item(), rel=1e-12)
    np.testing.assert_allclose(out["dH"], Ht_.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(out["dW"], Wt_.grad.numpy(), rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("partial", [True, False])
def test_topk_gradients_match_torch_autograd(partial):
    H, W, kw = _rand_case(3, N=9, d=5, V=23, K=5, mode="topk", partial=partial, T=1.4)
    g = 2.5
    out = oracle.kl_loss(H, W, grad_loss=g, **kw)
    Hq = torch.tensor(H, requires_grad=True)
    Wq = torch.tensor(W, requires_grad=True)
    idx = torch.tensor(kw["topk_idx"]).long()
    t = torch.tensor(kw["topk_logit"]) / 1.4
    if partial:
        q = torch.exp(t - torch.tensor(kw["teacher_lse"])[:, None])
    else:
        q = torch.softmax(t, dim=1)
    log_ps = torch.log_softmax(Hq @ Wq.T / 1.4, dim=1).gather(1, idx)
    rows = (q * (torch.log(q) - log_ps)).sum(1)
    keep = torch.tensor(kw["mask"]).bool()
    L = rows[keep].mean()
    (g * L).backward()
    assert out["loss"] == pytest.approx(L.item(), rel=1e-12)
    np.testing.assert_allclose(out["dH"], Hq.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(out["dW"], Wq.grad.numpy(), rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("beta", [1.0, 0.35])
def test_reverse_and_mixed_kl_match_scipy_and_torch_autograd(beta):
    H, W, kw = _rand_case(17, N=7, d=5, V=19, mode="hidden", masked=True, T=1.6)
    out = oracle.kl_loss(H, W, reverse_weight=beta, grad_loss=0.9, **kw)
    p_s = scipy.special.softmax(H @ W.T / 1.6, axis=1)
    p_t = scipy.special.softmax(kw["Ht"] @ kw["Wt"].T / 1.6, axis=1)
    keep = kw["mask"].astype(bool)
    for n in np.nonzero(keep)[0]:
        ref = (1 - beta) * scipy.stats.entropy(p_t[n], p_s[n]) + beta * scipy.stats.entropy(
            p_s[n], p_t[n])
        assert out["row_loss"][n] == pytest.approx(ref, rel=1e-11, abs=1e-14)
    Hq = torch.tensor(H, requires_grad=True)
    Wq = torch.tensor(W, requires_grad=True)
    log_ps = torch.log_softmax(Hq @ Wq.T / 1.6, dim=1)
    log_pt = torch.log_softmax(torch.tensor(kw["Ht"]) @ torch.tensor(kw["Wt"]).T / 1.6, dim=1)
    kl = torch.nn.functional.kl_div
    rows = ((1 - beta) * kl(log_ps, log_pt, reduction="none", log_target=True).sum(1)
            + beta * kl(log_pt, log_ps, reduction="none", log_target=True).sum(1))
    L = rows[torch.tensor(keep)].mean()
    (0.9 * L).backward()
    assert out["loss"] == pytest.approx(L.item(), rel=1e-12)
    np.testing.assert_allclose(out["dH"], Hq.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(out["dW"], Wq.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_reverse_weight_needs_teacher_hidden_mode():
    H, W, kw = _rand_case(18, mode="topk")
    with pytest.raises(ValueError):
        oracle.kl_loss(H, W, reverse_weight=0.5, **kw)


# ------------------------------------------------------------ finite differences

def _fd_check(H, W, kw, g=1.0, normalizer=None, h=1e-6):
    out = oracle.kl_loss(H, W, grad_loss=g, normalizer=normalizer, **kw)

    def L(Hx, Wx):
        o = oracle.kl_loss(Hx, Wx, grad_loss=g, normalizer=normalizer, want_dH=False,
                           want_dW=False, **kw)
        return g * float(np.sum(o["row_loss"])) / (normalizer or o["n_valid"])

    fdH = np.zeros_like(H)
    for i in np.ndindex(*H.shape):
        Hp, Hm = H.copy(), H.copy()
        Hp[i] += h
        Hm[i] -= h
        fdH[i] = (L(Hp, W) - L(Hm, W)) / (2 * h)
    fdW = np.zeros_like(W)
    for i in np.ndindex(*W.shape):
        Wp, Wm = W.copy(), W.copy()
        Wp[i] += h
        Wm[i] -= h
        fdW[i] = (L(H, Wp) - L(H, Wm)) / (2 * h)
    scale = max(np.max(np.abs(fdH)), np.max(np.abs(fdW)))
    return (max(np.max(np.abs(fdH - out["dH"])), np.max(np.abs(fdW - out["dW"]))) / scale)


@pytest.mark.parametrize("mode,partial", [("topk", True), ("topk", False), ("hidden", True)])
def test_finite_differences(mode, partial):
    H, W, kw = _rand_case(4, N=5, d=4, V=11, K=3, mode=mode, partial=partial, T=1.7)
    assert _fd_check(H, W, kw, g=0.7) < 1e-7


@pytest.mark.parametrize("beta", [1.0, 0.4])
def test_finite_differences_reverse_and_mixed(beta):
    H, W, kw = _rand_case(19, N=5, d=4, V=11, mode="hidden", T=1.7)
    kw = dict(kw, reverse_weight=beta)
    assert _fd_check(H, W, kw, g=0.8) < 1e-7


@pytest.mark.parametrize("mode,partial", [("topk", True), ("topk", False), ("hidden", True)])
def test_finite_differences_per_token_temperature(mode, partial):
    H, W, kw = _rand_case(20, N=5, d=4, V=11, K=3, mode=mode, partial=partial)
    Tr = np.array([0.7, 1.3, 2.1, 1.0, 0.9])
    kw = dict(kw, T=Tr)
    if mode == "topk" and partial:  # the cache's lse at each row's own temperature
        rng = np.random.default_rng(20)
        kw["teacher_lse"] = kw["teacher_lse"] + rng.normal(scale=0.1, size=5)
    assert _fd_check(H, W, kw, g=1.1) < 1e-7


def test_per_token_temperature_equals_rows_at_their_own_scalar_T():
    H, W, kw = _rand_case(21, N=6, d=4, V=13, K=4, mode="topk", masked=False)
    Tr = np.array([0.5, 1.0, 1.5, 2.0, 2.5, 3.0])
    t = kw["topk_logit"]
    both = oracle.kl_loss(H, W, **dict(kw, T=Tr))
    dW = np.zeros_like(W)
    for n in range(6):
        one = oracle.kl_loss(H[n:n + 1], W, T=float(Tr[n]), mode="topk",
                             topk_idx=kw["topk_idx"][n:n + 1], topk_logit=t[n:n + 1],
                             teacher_lse=kw["teacher_lse"][n:n + 1], normalizer=6)
        assert both["row_loss"][n] == pytest.approx(one["row_loss"][0], rel=1e-13)
        np.testing.assert_allclose(both["dH"][n], one["dH"][0], rtol=1e-12, atol=1e-16)
        dW += one["dW"]
    np.testing.assert_allclose(both["dW"], dW, rtol=1e-11, atol=1e-16)


def test_finite_differences_custom_normalizer():
    H, W, kw = _rand_case(5, N=4, d=3, V=9, K=3, mode="topk", T=0.9)
    assert _fd_check(H, W, kw, g=1.3, normalizer=11.0) < 1e-7


# ----------------------------------------------------------- K = V equivalences

@pytest.mark.parametrize("T", [1.0, 2.0])
def test_topk_with_K_equal_V_equals_full_kl(T):
    """With the whole vocabulary cached and the exact teacher lse, the partial-
    mass top-K loss is the full forward KL (and so is the renormalised one)."""
    H, W, kw = _rand_case(6, N=6, d=4, V=15, mode="hidden", T=T)
    full = oracle.kl_loss(H, W, **kw)
    t = kw["Ht"] @ kw["Wt"].T
    idx = np.tile(np.arange(15, dtype=np.int32), (6, 1))
    for lse in (scipy.special.logsumexp(t / T, axis=1), None):
        tk = oracle.kl_loss(H, W, T=T, mask=kw["mask"], mode="topk", topk_idx=idx,
                            topk_logit=t, teacher_lse=lse)
        assert tk["loss"] == pytest.approx(full["loss"], rel=1e-12)
        np.testing.assert_allclose(tk["dH"], full["dH"], rtol=1e-10, atol=1e-15)
        np.testing.assert_allclose(tk["dW"], full["dW"], rtol=1e-10, atol=1e-15)


def test_identical_teacher_gives_zero():
    H, W, kw = _rand_case(7, N=6, d=4, V=12, mode="hidden")
    out = oracle.kl_loss(H, W, T=1.3, mode="hidden", Ht=H, Wt=W)
    assert abs(out["loss"]) < 1e-14
    assert np.max(np.abs(out["dH"])) < 1e-14 and np.max(np.abs(out["dW"])) < 1e-14


def test_nonnegativity_and_partial_mass_bound():
    for seed in range(5):
        H, W, kw = _rand_case(10 + seed, mode="hidden", masked=False)
        assert np.all(oracle.kl_loss(H, W, **kw)["row_loss"] >= -1e-14)
        H, W, kw = _rand_case(20 + seed, mode="topk", partial=False, masked=False)
        assert np.all(oracle.kl_loss(H, W, **kw)["row_loss"] >= -1e-14)
        # Partial mass: by the log-sum inequality l >= m log(m / P_S) with P_S the
        # student's probability mass on the cached support; plain l >= 0 fails.
        H, W, kw = _rand_case(30 + seed, mode="topk", partial=True, masked=False)
        out = oracle.kl_loss(H, W, **kw)
        idx, q, _ = ko.teacher_support_probs(kw["topk_idx"], kw["topk_logit"], kw["T"],
                                             kw["teacher_lse"], W.shape[0])
        p_s = scipy.special.softmax(H @ W.T / kw["T"], axis=1)
        m = q.sum(1)
        P_S = np.take_along_axis(p_s, idx, axis=1).sum(1)
        assert np.all(out["row_loss"] >= m * np.log(m / P_S) - 1e-13)


# ------------------------------------------------------------- closed forms, W = 0

def test_W_zero_closed_forms():
    rng = np.random.default_rng(8)
    N, d, V, K, T = 5, 3, 10, 4, 1.5
    H = rng.normal(size=(N, d))
    W = np.zeros((V, d))
    t = rng.normal(size=(N, V))
    idx = np.argsort(-t, axis=1)[:, :K].astype(np.int32)
    logit = np.take_along_axis(t, idx, axis=1)
    lse_t = scipy.special.logsumexp(t / T, axis=1)
    out = oracle.kl_loss(H, W, T=T, mode="topk", topk_idx=idx, topk_logit=logit,
                         teacher_lse=lse_t)
    q = np.exp(logit / T - lse_t[:, None])
    m = q.sum(1)
    rows = (q * np.log(q)).sum(1) + m * np.log(V)
    assert out["loss"] == pytest.approx(rows.mean(), rel=1e-12)
    assert np.max(np.abs(out["dH"])) == 0.0
    dS = np.tile((m / V)[:, None], (1, V))
    for n in range(N):
        dS[n, idx[n]] -= q[n]
    dS /= (N * T)
    np.testing.assert_allclose(out["dW"], dS.T @ H, rtol=1e-12, atol=1e-15)
    # full mode with W = 0: KL = log V - entropy(p_t)
    Wt = rng.normal(size=(V, 2))
    Ht = rng.normal(size=(N, 2))
    full = oracle.kl_loss(H, W, T=T, mode="hidden", Ht=Ht, Wt=Wt)
    p_t = scipy.special.softmax(Ht @ Wt.T / T, axis=1)
    np.testing.assert_allclose(full["row_loss"],
                               np.log(V) - scipy.stats.entropy(p_t, axis=1), rtol=1e-12)


# ----------------------------------------------------------- dense reconstruction

@pytest.mark.parametrize("partial", [True, False])
def test_dense_reconstruction_equals_oracle(partial):
    H, W, kw = _rand_case(9, N=8, d=5, V=21, K=6, mode="topk", partial=partial, T=1.2)
    out = oracle.kl_loss(H, W, **kw)
    dense = oracle.dense_reconstruction_loss(H, W, T=kw["T"], topk_idx=kw["topk_idx"],
                                             topk_logit=kw["topk_logit"],
                                             teacher_lse=kw["teacher_lse"], mask=kw["mask"])
    assert out["loss"] == pytest.approx(dense, rel=1e-12)


# --------------------------------------------------------------------- invariants

def test_mask_equals_subset():
    H, W, kw = _rand_case(11, N=9, d=4, V=14, K=4, mode="topk", masked=True)
    out = oracle.kl_loss(H, W, **kw)
    keep = kw["mask"].astype(bool)
    sub = oracle.kl_loss(H[keep], W, T=kw["T"], mode="topk", topk_idx=kw["topk_idx"][keep],
                         topk_logit=kw["topk_logit"][keep], teacher_lse=kw["teacher_lse"][keep])
    assert out["loss"] == pytest.approx(sub["loss"], rel=1e-13)
    np.testing.assert_allclose(out["dW"], sub["dW"], rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(out["dH"][keep], sub["dH"], rtol=1e-12, atol=1e-16)
    assert np.all(out["dH"][~keep] == 0) and np.all(out["row_loss"][~keep] == 0)


def test_no_valid_rows_gives_zero():
    H, W, kw = _rand_case(12, mode="topk")
    kw["mask"] = np.zeros(H.shape[0], dtype=np.uint8)
    out = oracle.kl_loss(H, W, **kw)
    assert out["loss"] == 0.0 and not np.any(out["dH"]) and not np.any(out["dW"])


def test_empty_slot_equals_dropped_entry_and_order_is_irrelevant():
    H, W, kw = _rand_case(13, N=5, d=3, V=12, K=4, mode="topk")
    base = oracle.kl_loss(H, W, **kw)
    rng = np.random.default_rng(0)
    perm = np.stack([rng.permutation(4) for _ in range(5)])
    kp = dict(kw, topk_idx=np.take_along_axis(kw["topk_idx"], perm, 1),
              topk_logit=np.take_along_axis(kw["topk_logit"], perm, 1))
    o2 = oracle.kl_loss(H, W, **kp)
    assert o2["loss"] == pytest.approx(base["loss"], rel=1e-13)
    np.testing.assert_allclose(o2["dW"], base["dW"], rtol=1e-12, atol=1e-16)
    # An extra empty slot (-1, arbitrary logit) changes nothing.
    ke = dict(kw, topk_idx=np.concatenate([kw["topk_idx"], -np.ones((5, 1), np.int32)], 1),
              topk_logit=np.concatenate([kw["topk_logit"], np.full((5, 1), 9.0)], 1))
    o3 = oracle.kl_loss(H, W, **ke)
    assert o3["loss"] == pytest.approx(base["loss"], rel=1e-13)
    np.testing.assert_allclose(o3["dH"], base["dH"], rtol=1e-12, atol=1e-16)


def test_temperature_scaling_identity():
    """s~ = s / T, so the loss at temperature T with inputs (H, t) equals the loss
    at T = 1 with (H / T, t / T); dW is unchanged and dH scales by 1/T."""
    T = 2.3
    for mode in ("topk", "hidden"):
        H, W, kw = _rand_case(14, N=5, d=4, V=11, K=3, mode=mode, T=T)
        a = oracle.kl_loss(H, W, **kw)
        k1 = dict(kw, T=1.0)
        if mode == "topk":
            k1["topk_logit"] = kw["topk_logit"] / T
        else:
            k1["Ht"] = kw["Ht"] / T
        b = oracle.kl_loss(H / T, W, **k1)
        assert a["loss"] == pytest.approx(b["loss"], rel=1e-12)
        np.testing.assert_allclose(a["dW"], b["dW"], rtol=1e-11, atol=1e-16)
        np.testing.assert_allclose(a["dH"], b["dH"] / T, rtol=1e-11, atol=1e-16)


def test_row_and_vocab_sampling_match_full_evaluation():
    H, W, kw = _rand_case(15, N=11, d=4, V=17, K=5, mode="topk")
    full = oracle.kl_loss(H, W, **kw)
    rows = np.array([0, 3, 10, 7])
    vr = np.array([16, 2, 5])
    part = oracle.kl_loss(H, W, rows=rows, vocab_rows=vr, **kw)
    np.testing.assert_allclose(part["row_loss"], full["row_loss"][rows], rtol=1e-14)
    np.testing.assert_allclose(part["lse_s"], full["lse_s"][rows], rtol=1e-14)
    np.testing.assert_allclose(part["dH"], full["dH"][rows], rtol=1e-13, atol=1e-17)
    np.testing.assert_allclose(part["dW"], full["dW"][vr], rtol=1e-12, atol=1e-17)


def test_invalid_cache_indices_raise():
    H, W, kw = _rand_case(16, mode="topk", K=3)
    bad = kw["topk_idx"].copy()
    bad[0, 0] = W.shape[0]
    with pytest.raises(ValueError):
        oracle.kl_loss(H, W, **dict(kw, topk_idx=bad))
    dup = kw["topk_idx"].copy()
    dup[1, 1] = dup[1, 0]
    with pytest.raises(ValueError):
        oracle.kl_loss(H, W, **dict(kw, topk_idx=dup))


# ------------------------------------------------------------------ planted mistakes

def _patched(monkeypatch, name, fn):
    monkeypatch.setattr(ko, name, fn)


def test_planted_mistakes_are_caught(monkeypatch):
    """Each planted mistake in the oracle is caught by one of the pins above."""
    orig_grad_topk = ko.grad_topk_rows
    orig_kl_topk = ko.kl_topk_rows
    orig_lse = ko.logsumexp_rows
    orig_scaled = ko.scaled_logits
    H, W, kw = _rand_case(4, N=5, d=4, V=11, K=3, mode="topk", T=1.7)
    goldens = _golden_cases()

    def golden_fails():
        try:
            for c in goldens:
                test_golden_closed_forms(c)
        except AssertionError:
            return True
        return False

    # 1. dropped mass factor m in the gradient
    _patched(monkeypatch, "grad_topk_rows",
             lambda s, l, i, q, v, T: orig_grad_topk(s, l, i, q / q.sum(1, keepdims=True), v, T)
             * 1.0)
    assert _fd_check(H, W, kw) > 1e-3
    monkeypatch.undo()
    # 2. wrong sign of the teacher term in the gradient
    def bad_sign(s, l, i, q, v, T):
        p = np.exp(s - l[:, None])
        g = q.sum(1)[:, None] * p
        r = np.arange(i.shape[0])
        for k in range(i.shape[1]):
            g[r[v[:, k]], i[v[:, k], k]] += q[v[:, k], k]
        return g / T
    _patched(monkeypatch, "grad_topk_rows", bad_sign)
    assert _fd_check(H, W, kw) > 1e-3
    monkeypatch.undo()
    # 3. dropped mass term m * lse_s from the loss
    _patched(monkeypatch, "kl_topk_rows",
             lambda s, l, i, q, v: orig_kl_topk(s, np.zeros_like(l), i, q, v))
    assert golden_fails()
    monkeypatch.undo()
    # 4. log-sum-exp missing its max shift back
    _patched(monkeypatch, "logsumexp_rows", lambda x: orig_lse(x) - np.max(x, axis=1))
    assert golden_fails()
    monkeypatch.undo()
    # 5. temperature applied twice / transposed head
    _patched(monkeypatch, "scaled_logits", lambda X, Wh, T: orig_scaled(X, Wh, T) / T)
    assert golden_fails()
    monkeypatch.undo()
    _patched(monkeypatch, "scaled_logits",
             lambda X, Wh, T: (X[:, ::-1] @ Wh.T) / T)
    assert _fd_check(H, W, kw) > 1e-3
    monkeypatch.undo()
