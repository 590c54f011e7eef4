"""Build the sm_100a shared library in-tree: chunked_kl_loss_tma_b200/libchunkedkl.so.

    python -m chunked_kl_loss_tma_b200.build [--verbose-ptxas]

The CUDA runtime is linked statically and the driver's tensor-map encoder is
resolved at run time, so the library also loads on a machine without a GPU
driver (its entry points then return an error)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "kl_api.cu")
OUT = os.path.join(HERE, "libchunkedkl.so")
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))]
DEPS.append(os.path.join(ROOT, "include", "chunked_kl.h"))


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def up_to_date():
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS + [__file__])


def build(force=False, verbose_ptxas=False):
    if not force and not verbose_ptxas and up_to_date():
        return OUT
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", OUT + ".tmp", SRC]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
