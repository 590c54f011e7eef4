"""The library from plain C on the GPU: tests/c_fwd_bwd.c allocates device
memory and runs kl_fwd_bwd with the CUDA runtime alone (no PyTorch in that
process), on a seeded bf16 top-K problem written to raw files.  Its loss and
gradients must match the fp64 oracle (loss relative error <= 1e-3, gradients
max-abs error <= 2e-2 max|oracle|) and, bit for bit, the Python binding's call
on the same inputs (the same kernels in the same order)."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_tma_b200 import build as B
from chunked_kl_loss_tma_b200 import ops
from chunked_kl_loss_tma_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    here = os.path.dirname(__file__)
    libdir = os.path.dirname(B.build())
    exe = str(tmp_path / "c_fwd_bwd")
    subprocess.run([cc, "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(os.path.dirname(here), "include"),
                    "-I", os.path.join(CUDA, "include"), os.path.join(here, "c_fwd_bwd.c"),
                    "-L", libdir, "-lchunkedkl", "-Wl,-rpath," + libdir,
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", exe],
                   check=True, capture_output=True, text=True)
    return exe


def test_fwd_bwd_from_plain_c(tmp_path):
    exe = _compile(tmp_path)
    N, d, V, K, T = 300, 136, 3001, 16, 1.3
    w = wl.make_topk("c_caller", N=N, d=d, V=V, K=K, d_t=64, T=T, dtype=torch.bfloat16,
                     w_std=0.08, tw_std=0.1, seed=95)
    raw = {"H.bin": w.H.view(torch.int16), "W.bin": w.W.view(torch.int16),
           "idx.bin": w.topk_idx, "val.bin": w.topk_logit, "lse.bin": w.teacher_lse}
    for name, t in raw.items():
        t.contiguous().numpy().tofile(tmp_path / name)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", "0"))
    r = subprocess.run([exe, str(tmp_path), str(N), str(d), str(V), str(K), repr(T)],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert (tmp_path / "status.txt").read_text().strip() == "0"
    loss = float(np.fromfile(tmp_path / "loss.bin", dtype=np.float32)[0])
    dH = torch.from_numpy(np.fromfile(tmp_path / "dH.bin", dtype=np.int16)).view(
        torch.bfloat16).reshape(N, d)
    dW = torch.from_numpy(np.fromfile(tmp_path / "dW.bin", dtype=np.float32)).reshape(V, d)

    ref = oracle.kl_loss(w.H, w.W, T=T, mode="topk", topk_idx=w.topk_idx,
                         topk_logit=w.topk_logit, teacher_lse=w.teacher_lse)
    assert abs(loss - ref["loss"]) <= 1e-3 * abs(ref["loss"])
    for name, got in (("dH", dH), ("dW", dW)):
        err = np.max(np.abs(got.double().numpy() - ref[name]))
        assert err <= 2e-2 * np.max(np.abs(ref[name])), (name, err)

    g = w.to("cuda")
    py = ops.kl_fwd_bwd(g.H, g.W, T=T, topk_idx=g.topk_idx, topk_logit=g.topk_logit,
                        teacher_lse=g.teacher_lse)
    assert np.float32(loss) == np.float32(py["loss"].item())
    assert torch.equal(dH, py["dH"].cpu())
    assert torch.equal(dW, py["dW"].cpu())
