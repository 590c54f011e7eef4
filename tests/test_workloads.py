"""Seeded input generators: deterministic, right shapes, and a teacher cache that
really is the teacher's top-K with its full-vocabulary log-sum-exp."""
import numpy as np
import torch

from chunked_kl_loss_tma_b200 import workloads as wl


def test_tiny_is_deterministic_and_shaped():
    a = wl.tiny()
    b = wl.tiny()
    assert a.H.shape == (64, 64) and a.W.shape == (1000, 64) and a.dtype == torch.float32
    assert a.topk_idx.shape == (64, 8) and a.topk_idx.dtype == torch.int32
    assert torch.equal(a.H, b.H) and torch.equal(a.topk_idx, b.topk_idx)
    assert abs(a.W.std().item() - 0.05) < 0.005 and abs(a.H.std().item() - 1.0) < 0.05


def test_teacher_cache_is_topk_with_full_lse():
    g = torch.Generator().manual_seed(5)
    Ht = torch.randn(7, 6, generator=g)
    Wt = torch.randn(40, 6, generator=g)
    idx, val, lse = wl.teacher_topk_cache(Ht, Wt, K=5, T=1.5, rows_per_block=3)
    t = (Ht.double() @ Wt.double().T).numpy()
    for n in range(7):
        order = np.argsort(-t[n])[:5]
        assert sorted(order.tolist()) == sorted(idx[n].tolist())
        np.testing.assert_allclose(val[n].numpy(), t[n][idx[n].long().numpy()], rtol=1e-5)
    ref = np.log(np.exp(t / 1.5).sum(1))
    np.testing.assert_allclose(lse.numpy(), ref, rtol=1e-6)


def test_packed_mask_counts():
    mask, lens = wl.packed_mask(32768, 0.05, seed=3)
    assert int((mask == 0).sum()) == round(0.05 * 32768)
    assert sum(lens) == 32768 and all(l <= 4096 for l in lens)
    assert all(512 <= l for l in lens[:-1])
