"""Bounded waits: a kernel whose waits run out records KL_ERR_TIMEOUT in the
status word, drains its in-flight copies and MMAs, releases TMEM and returns,
and the CUDA context stays usable.  The test forces every wait to run out by
setting the spin limit (KL_SPIN_LIMIT, read once per process) to one clock
cycle in a child process; nothing faults, traps or hangs."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    from chunked_kl_loss_tma_b200 import ops, workloads as wl
    w = wl.make_topk("wd", N=600, d=256, V=9000, K=16, d_t=64, T=1.0,
                     dtype=torch.bfloat16, w_std=0.05, tw_std=0.1, seed=41).to("cuda")
    codes = []
    for fuse in (False, True):  # the separate dlogits pass, and dS formed inside dH
        out = ops.kl_fwd_bwd(w.H, w.W, topk_idx=w.topk_idx, topk_logit=w.topk_logit,
                             teacher_lse=w.teacher_lse, chunk_tokens=256, fuse_dlogits=fuse)
        codes.append(ops.status(out["workspace"]))
    torch.cuda.synchronize()
    ok = float(torch.ones(1000, device="cuda").sum().item()) == 1000.0
    print("STATUS", codes[0], codes[1], "CONTEXT_OK", ok)
""")


def _run(limit):
    env = dict(os.environ, KL_SPIN_LIMIT=str(limit))
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [l for l in r.stdout.splitlines() if l.startswith("STATUS")][-1].split()
    return int(line[1]), int(line[2]), line[4] == "True"


def test_waits_that_run_out_report_timeout_and_keep_the_context():
    a, b, ok = _run(1)
    assert a == 8 and b == 8 and ok  # KL_ERR_TIMEOUT twice, context still usable


def test_default_limit_does_not_time_out():
    a, b, ok = _run(0)  # 0 = library default
    assert a == 0 and b == 0 and ok
