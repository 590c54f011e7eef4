"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, sizes workspaces as O(chunk * V + N), and rejects bad
arguments on the host before touching a device."""
import os
import re

import pytest

from chunked_kl_loss_tma_b200 import _lib as L
from chunked_kl_loss_tma_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "chunked_kl.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_\s\*]*?\b(kl_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_functions():
    assert _declared() == sorted(L.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def _problem(**kw):
    p = L.KLProblem()
    p.N, p.d, p.V, p.dtype, p.teacher, p.K, p.T = 4096, 3072, 128256, 0, 0, 64, 1.0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_workspace_is_chunk_sized_not_NV(lib):
    small = L.kl_workspace_bytes(_problem(N=4096), L.KL_ENTRY_FWD_BWD)
    big = L.kl_workspace_bytes(_problem(N=262144), L.KL_ENTRY_FWD_BWD)
    # one [4096, V] bf16 logit chunk + per-chunk stats; growth with N is O(N) only
    assert small >= 4096 * 128256 * 2
    assert big - small <= (262144 - 4096) * 8 + 4096
    assert big < 262144 * 128256 * 2 / 10
    assert L.kl_workspace_bytes(_problem(chunk_tokens=1024), 2) < small


def test_workspace_hidden_mode_has_two_logit_buffers(lib):
    p = _problem(teacher=1, d_t=4096, K=0)
    assert L.kl_workspace_bytes(p, 2) >= 2 * 4096 * 128256 * 2


@pytest.mark.parametrize("field,value,code", [
    ("d", 3070, 4),           # rows not 16-byte aligned -> KL_ERR_ALIGN
    ("dtype", 7, 3),          # KL_ERR_DTYPE
    ("teacher", 5, 3),
    ("K", 0, 2),              # KL_ERR_SHAPE
    ("K", 1025, 2),
    ("V", 0, 2),
    ("N", -1, 2),
    ("T", 0.0, 10),           # KL_ERR_ARG
    ("T", -1.0, 10),
    ("chunk_tokens", -5, 10),
    ("reverse_weight", 0.5, 10),   # reverse KL needs the teacher-hidden mode
    ("reverse_weight", -0.1, 10),
])
def test_bad_problems_rejected_on_host(lib, field, value, code):
    p = _problem(**{field: value})
    assert L.kl_workspace_bytes(p, 2) == 0
    p.H = p.W = p.topk_idx = p.topk_logit = 256
    rc = L.kl_fwd_bwd(p, 256, 1 << 40, 1.0, 256, None, 256, 256, 0, None)
    assert rc == code, (rc, L.kl_status_string(rc))


def test_reverse_weight_range_in_hidden_mode(lib):
    p = _problem(teacher=1, d_t=4096, K=0, reverse_weight=1.0)
    assert L.kl_workspace_bytes(p, 2) > 0
    p.reverse_weight = 1.5
    assert L.kl_workspace_bytes(p, 2) == 0


def test_null_and_misaligned_pointers_rejected(lib):
    p = _problem()
    assert L.kl_fwd_bwd(p, 256, 1 << 40, 1.0, 256, None, 256, 256, 0, None) == 1
    p.H, p.W, p.topk_idx, p.topk_logit = 264, 256, 256, 256
    assert L.kl_fwd_bwd(p, 256, 1 << 40, 1.0, 256, None, 256, 256, 0, None) == 4
    p.H = 272
    # valid arguments: without a CUDA device the call fails with KL_ERR_CUDA
    import torch
    if not torch.cuda.is_available():
        assert L.kl_fwd_bwd(p, 256, 1 << 40, 1.0, 256, None, 256, 256, 0, None) == 6


def test_status_strings(lib):
    for code, name in L.STATUS.items():
        assert L.kl_status_string(code) and isinstance(L.kl_status_string(code), str)
    assert lib.kl_launch_count() >= 0


def test_vocab_parallel_host_checks(lib):
    p = _problem(chunk_tokens=1024, v_begin=1024, V=4096, V_total=128256)
    assert L.kl_vp_num_chunks(p) == 4
    assert L.kl_vp_num_chunks(_problem(N=0, V_total=128256)) == 0
    assert L.kl_vp_num_chunks(_problem(v_begin=256, V_total=128256)) == -1   # past the head
    assert L.kl_vp_num_chunks(_problem(v_begin=-1, V_total=128256)) == -1
    assert L.kl_vp_num_chunks(_problem(v_begin=8)) == -1                     # shard without V_total
    p.H = p.W = p.topk_idx = p.topk_logit = 256
    # the whole-head entry points refuse a shard
    assert L.kl_fwd_bwd(p, 256, 1 << 40, 1.0, 256, None, 256, 256, 0, None) == 10
    assert L.kl_fwd(p, 256, 1 << 40, 256, 256, None, None, None) == 10
    # chunk index, rank and reverse weight are checked before the device
    assert L.kl_vp_fwd_chunk(p, 4, 256, 1 << 40, 256, None) == 10
    assert L.kl_vp_fwd_chunk(p, -1, 256, 1 << 40, 256, None) == 10
    assert L.kl_vp_bwd_chunk(p, 0, 256, 1 << 40, 256, None, 2, 2, 1.0, 256, None, None, 256,
                             256, 0, None) == 10
    assert L.kl_vp_bwd_chunk(p, 0, 256, 1 << 40, 256, None, 0, 0, 1.0, 256, None, None, 256,
                             256, 0, None) == 10
    # the middle phase exists for the teacher-hidden mode only
    assert L.kl_vp_mid_chunk(p, 0, 256, 1 << 40, 256, 2, 0, 256, None) == 10
    q = _problem(teacher=1, d_t=4096, K=0, V=4096, V_total=128256, reverse_weight=0.5)
    q.H = q.W = q.Ht = q.Wt = 256
    assert L.kl_vp_mid_chunk(q, 0, 256, 1 << 40, 256, 0, 0, 256, None) == 10   # P < 1
    assert L.kl_vp_mid_chunk(q, 9, 256, 1 << 40, 256, 2, 1, 256, None) == 10   # no chunk 9


def test_cast_host_checks(lib):
    assert L.kl_cast_f32(256, 256, 6, L.KL_DTYPE_BF16, None) == 2      # n not a multiple of 4
    assert L.kl_cast_f32(256, 256, 8, 9, None) == 3
    assert L.kl_cast_f32(None, 256, 8, L.KL_DTYPE_BF16, None) == 1
    assert L.kl_cast_f32(260, 256, 8, L.KL_DTYPE_BF16, None) == 4
    assert L.kl_cast_f32(None, None, 0, L.KL_DTYPE_BF16, None) == 0


def test_keep_last_chunk_flag_rules(lib):
    """keep_last_chunk: 0 or 1; one workspace layout for every entry (kl_fwd
    leaves the chunk where kl_bwd reads it); refused by the calls that do not
    pass a chunk from a forward to a backward."""
    p = _problem()
    sizes = [L.kl_workspace_bytes(p, e) for e in (0, 1, 2)]
    p.keep_last_chunk = 1
    kept = [L.kl_workspace_bytes(p, e) for e in (0, 1, 2)]
    assert kept[0] == kept[1] == kept[2] == sizes[2]
    p.keep_last_chunk = 2
    assert L.kl_workspace_bytes(p, 0) == 0
    p.keep_last_chunk = 1
    dummy = 1 << 20
    rc = L.kl_fwd_bwd(p, dummy, kept[2], 1.0, dummy, None, dummy, dummy, 0, None)
    assert rc == 10  # KL_ERR_ARG
    rc = L.kl_fwd_noalloc(p, dummy, dummy, dummy, None, None)
    assert rc == 10


def test_fuse_dlogits_flag_rules(lib):
    """fuse_dlogits: 0 or 1; the fused pass's workspace grows by one chunk of dS
    (bf16 top-K only); kl_fwd, kl_bwd and the no-allocation forward refuse it."""
    p = _problem()
    base = L.kl_workspace_bytes(p, 2)
    p.fuse_dlogits = 1
    assert L.kl_workspace_bytes(p, 2) >= base + 4096 * 128256 * 2
    p.dtype = 1  # fp32 inputs keep the dlogits pass: no extra buffer
    assert L.kl_workspace_bytes(p, 2) == L.kl_workspace_bytes(_problem(dtype=1), 2)
    p.dtype = 0
    p.fuse_dlogits = 2
    assert L.kl_workspace_bytes(p, 2) == 0
    p.fuse_dlogits = 1
    dummy = 1 << 20
    assert L.kl_fwd(p, dummy, base, dummy, dummy, None, None, None) == 10  # KL_ERR_ARG
    assert L.kl_bwd(p, dummy, base, dummy, None, dummy, dummy, dummy, 0, None) == 10
    assert L.kl_fwd_noalloc(p, dummy, dummy, dummy, None, None) == 10


def test_plain_c_caller(lib, tmp_path):
    """The header compiles as strict C99, the library links from C, and a C
    caller gets the answers the Python binding gets (tests/abi_c_caller.c)."""
    import ctypes
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    here = os.path.dirname(__file__)
    libdir = os.path.dirname(B.OUT)
    exe = str(tmp_path / "abi_c_caller")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.dirname(HEADER), os.path.join(here, "abi_c_caller.c"),
                    "-L", libdir, "-lchunkedkl", "-Wl,-rpath," + libdir, "-o", exe],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(got["sizeof_problem"]) == ctypes.sizeof(L.KLProblem)
    for e in (L.KL_ENTRY_FWD, L.KL_ENTRY_BWD, L.KL_ENTRY_FWD_BWD):
        assert int(got[f"ws_topk_{e}"]) == L.kl_workspace_bytes(_problem(), e)
    hidden = _problem(teacher=1, K=0, d_t=4096, N=8192, T=2.0)
    assert int(got["ws_hidden"]) == L.kl_workspace_bytes(hidden, L.KL_ENTRY_FWD_BWD)
    code = {name: c for c, name in L.STATUS.items()}
    assert int(got["ws_bad_T"]) == 0
    assert int(got["fwd_bwd_bad_T"]) == code["KL_ERR_ARG"]
    assert int(got["fwd_bwd_bad_d"]) == code["KL_ERR_ALIGN"]
    assert int(got["fwd_null_inputs"]) == code["KL_ERR_NULL"]
    assert int(got["fwd_bwd_null"]) == code["KL_ERR_NULL"]
    assert got["status_string_align"] == L.kl_status_string(code["KL_ERR_ALIGN"])
    assert int(got["noalloc_scratch"]) == L.KL_NOALLOC_SCRATCH_BYTES

