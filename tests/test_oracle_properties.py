"""Property checks of the fp64 oracle over random small shapes (hypothesis).

The pins in test_oracle_pins.py fix the oracle on hand-picked sizes; these draw
the sizes, temperatures, masks and cache widths at random and check what the
mathematics forces at every size: the identity teacher gives zero loss and zero
gradient, the full KL is non-negative, the top-K loss with K = V and the exact
teacher normaliser equals the full-vocabulary KL, the renormalised top-K loss
is at least -log of the student's mass on the support, the result does not
depend on how many rows the oracle evaluates per block, and the gradient of H
matches central finite differences."""
import numpy as np
import scipy.special
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=25, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    N = draw(st.integers(1, 7))
    d = draw(st.integers(1, 6))
    V = draw(st.integers(2, 24))
    K = draw(st.integers(1, V))
    T = draw(st.floats(0.3, 4.0))
    seed = draw(st.integers(0, 2**31 - 1))
    masked = draw(st.booleans())
    rng = np.random.default_rng(seed)
    H = rng.normal(size=(N, d))
    W = rng.normal(scale=0.8, size=(V, d))
    Ht = rng.normal(size=(N, d))
    Wt = rng.normal(scale=0.8, size=(V, d))
    mask = None
    if masked:
        mask = (rng.random(N) > 0.3).astype(np.uint8)
        mask[0] = 1  # at least one row in the mean
    return dict(N=N, d=d, V=V, K=K, T=T, H=H, W=W, Ht=Ht, Wt=Wt, mask=mask)


def _cache(p, K):
    t = p["Ht"] @ p["Wt"].T
    idx = np.argsort(-t, axis=1)[:, :K].astype(np.int32)
    return idx, np.take_along_axis(t, idx, axis=1), scipy.special.logsumexp(t / p["T"], axis=1)


@SETTINGS
@given(problems())
def test_identity_teacher_gives_zero_loss_and_gradient(p):
    o = oracle.kl_loss(p["H"], p["W"], T=p["T"], mask=p["mask"], mode="hidden", Ht=p["H"],
                       Wt=p["W"])
    assert abs(o["loss"]) < 1e-12
    assert np.max(np.abs(o["dH"])) < 1e-12 and np.max(np.abs(o["dW"])) < 1e-12


@SETTINGS
@given(problems())
def test_full_kl_is_nonnegative_per_row(p):
    o = oracle.kl_loss(p["H"], p["W"], T=p["T"], mask=p["mask"], mode="hidden", Ht=p["Ht"],
                       Wt=p["Wt"])
    assert np.min(o["row_loss"]) > -1e-12


@SETTINGS
@given(problems())
def test_topk_with_all_entries_equals_full_kl(p):
    idx, logit, lse = _cache(p, p["V"])
    full = oracle.kl_loss(p["H"], p["W"], T=p["T"], mask=p["mask"], mode="hidden", Ht=p["Ht"],
                          Wt=p["Wt"])
    for teacher_lse in (lse, None):  # partial mass with K = V, and renormalised
        tk = oracle.kl_loss(p["H"], p["W"], T=p["T"], mask=p["mask"], mode="topk",
                            topk_idx=idx, topk_logit=logit, teacher_lse=teacher_lse)
        np.testing.assert_allclose(tk["row_loss"], full["row_loss"], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(tk["dH"], full["dH"], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(tk["dW"], full["dW"], rtol=1e-9, atol=1e-12)


@SETTINGS
@given(problems())
def test_renormalised_topk_is_at_least_minus_log_support_mass(p):
    idx, logit, _ = _cache(p, p["K"])
    o = oracle.kl_loss(p["H"], p["W"], T=p["T"], mode="topk", topk_idx=idx, topk_logit=logit,
                       teacher_lse=None)
    s = p["H"] @ p["W"].T / p["T"]
    logp = s - scipy.special.logsumexp(s, axis=1, keepdims=True)
    mass = np.exp(np.take_along_axis(logp, idx, axis=1)).sum(1)
    assert np.all(o["row_loss"] >= -np.log(mass) - 1e-10)


@SETTINGS
@given(problems(), st.integers(1, 4))
def test_block_size_does_not_change_the_result(p, block):
    idx, logit, lse = _cache(p, p["K"])
    kw = dict(T=p["T"], mask=p["mask"], mode="topk", topk_idx=idx, topk_logit=logit,
              teacher_lse=lse)
    a = oracle.kl_loss(p["H"], p["W"], block=block, **kw)
    b = oracle.kl_loss(p["H"], p["W"], block=256, **kw)
    np.testing.assert_allclose(a["row_loss"], b["row_loss"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a["dW"], b["dW"], rtol=1e-12, atol=1e-14)


@SETTINGS
@given(problems(), st.sampled_from(["topk", "hidden"]))
def test_dH_matches_central_differences(p, mode):
    idx, logit, lse = _cache(p, p["K"])
    kw = dict(T=p["T"], mask=p["mask"], mode=mode)
    if mode == "topk":
        kw.update(topk_idx=idx, topk_logit=logit, teacher_lse=lse)
    else:
        kw.update(Ht=p["Ht"], Wt=p["Wt"])
    o = oracle.kl_loss(p["H"], p["W"], **kw)
    h = 1e-5
    n, j = 0, p["d"] - 1
    Hp, Hm = p["H"].copy(), p["H"].copy()
    Hp[n, j] += h
    Hm[n, j] -= h
    fd = (oracle.kl_loss(Hp, p["W"], want_dH=False, want_dW=False, **kw)["loss"] -
          oracle.kl_loss(Hm, p["W"], want_dH=False, want_dW=False, **kw)["loss"]) / (2 * h)
    assert abs(fd - o["dH"][n, j]) <= 1e-6 * max(1.0, abs(fd))
