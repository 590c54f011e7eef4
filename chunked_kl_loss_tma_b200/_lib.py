"""ctypes binding of libchunkedkl.so (argument marshalling only).

Every computation runs in the library's CUDA kernels.  There is no fallback:
if the library is missing or the device is not sm_100, calls raise."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libchunkedkl.so")

KL_DTYPE_BF16 = 0
KL_DTYPE_F32 = 1
KL_TEACHER_TOPK = 0
KL_TEACHER_HIDDEN = 1
KL_ENTRY_FWD = 0
KL_ENTRY_BWD = 1
KL_ENTRY_FWD_BWD = 2

STATUS = {
    0: "KL_OK", 1: "KL_ERR_NULL", 2: "KL_ERR_SHAPE", 3: "KL_ERR_DTYPE", 4: "KL_ERR_ALIGN",
    5: "KL_ERR_WORKSPACE", 6: "KL_ERR_CUDA", 7: "KL_ERR_INDEX", 8: "KL_ERR_TIMEOUT",
    9: "KL_ERR_UNSUPPORTED", 10: "KL_ERR_ARG", 11: "KL_ERR_TOO_LARGE",
}
KL_NOALLOC_SCRATCH_BYTES = 16 << 20

# Every symbol declared in include/chunked_kl.h.
EXPORTS = ("kl_workspace_bytes", "kl_fwd", "kl_bwd", "kl_fwd_bwd", "kl_status",
           "kl_status_string", "kl_launch_count", "kl_profile_begin", "kl_profile_end",
           "kl_fwd_noalloc", "kl_vp_num_chunks", "kl_vp_fwd_chunk", "kl_vp_mid_chunk",
           "kl_vp_bwd_chunk", "kl_cast_f32")


class KLProblem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64), ("d", ctypes.c_int64), ("V", ctypes.c_int64),
        ("dtype", ctypes.c_int32), ("teacher", ctypes.c_int32),
        ("H", ctypes.c_void_p), ("W", ctypes.c_void_p), ("mask", ctypes.c_void_p),
        ("T", ctypes.c_float), ("K", ctypes.c_int32),
        ("topk_idx", ctypes.c_void_p), ("topk_logit", ctypes.c_void_p),
        ("teacher_lse", ctypes.c_void_p),
        ("d_t", ctypes.c_int64), ("Ht", ctypes.c_void_p), ("Wt", ctypes.c_void_p),
        ("chunk_tokens", ctypes.c_int64), ("normalizer", ctypes.c_float),
        ("reverse_weight", ctypes.c_float), ("T_row", ctypes.c_void_p),
        ("v_begin", ctypes.c_int64), ("V_total", ctypes.c_int64),
        ("keep_last_chunk", ctypes.c_int32), ("fuse_dlogits", ctypes.c_int32),
    ]


class KLProfileEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_uint64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


class KLError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({_string(code)})")


_lib = None


def lib():
    """Load the library once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m chunked_kl_loss_tma_b200.build` (no fallback path exists)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(KLProblem)
    vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    L.kl_workspace_bytes.argtypes = [P, i32]
    L.kl_workspace_bytes.restype = sz
    L.kl_fwd.argtypes = [P, vp, sz, vp, vp, vp, vp, vp]
    L.kl_fwd.restype = i32
    L.kl_bwd.argtypes = [P, vp, sz, vp, vp, vp, vp, vp, i32, vp]
    L.kl_bwd.restype = i32
    L.kl_fwd_bwd.argtypes = [P, vp, sz, f32, vp, vp, vp, vp, i32, vp]
    L.kl_fwd_bwd.restype = i32
    L.kl_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp]
    L.kl_fwd_noalloc.restype = i32
    i64 = ctypes.c_int64
    L.kl_vp_num_chunks.argtypes = [P]
    L.kl_vp_num_chunks.restype = i64
    L.kl_vp_fwd_chunk.argtypes = [P, i64, vp, sz, vp, vp]
    L.kl_vp_fwd_chunk.restype = i32
    L.kl_vp_mid_chunk.argtypes = [P, i64, vp, sz, vp, i32, i32, vp, vp]
    L.kl_vp_mid_chunk.restype = i32
    L.kl_vp_bwd_chunk.argtypes = [P, i64, vp, sz, vp, vp, i32, i32, f32, vp, vp, vp, vp, vp, i32,
                                  vp]
    L.kl_vp_bwd_chunk.restype = i32
    L.kl_cast_f32.argtypes = [vp, vp, i64, i32, vp]
    L.kl_cast_f32.restype = i32
    L.kl_status.argtypes = [vp, vp]
    L.kl_status.restype = i32
    L.kl_status_string.argtypes = [i32]
    L.kl_status_string.restype = ctypes.c_char_p
    L.kl_launch_count.argtypes = []
    L.kl_launch_count.restype = ctypes.c_uint64
    L.kl_profile_begin.argtypes = []
    L.kl_profile_begin.restype = i32
    L.kl_profile_end.argtypes = [ctypes.POINTER(KLProfileEntry), i32]
    L.kl_profile_end.restype = i32
    _lib = L
    return L


def _string(code):
    try:
        return lib().kl_status_string(int(code)).decode()
    except Exception:  # pragma: no cover
        return "?"


def check(code, where):
    if code != 0:
        raise KLError(code, where)


def kl_workspace_bytes(prob, entry):
    return lib().kl_workspace_bytes(ctypes.byref(prob), entry)


def kl_fwd(prob, ws, ws_bytes, loss, lse_s, lse_t, row_loss, stream):
    return lib().kl_fwd(ctypes.byref(prob), ws, ws_bytes, loss, lse_s, lse_t, row_loss, stream)


def kl_bwd(prob, ws, ws_bytes, lse_s, lse_t, grad_loss, dH, dW, accumulate_dW, stream):
    return lib().kl_bwd(ctypes.byref(prob), ws, ws_bytes, lse_s, lse_t, grad_loss, dH, dW,
                        int(accumulate_dW), stream)


def kl_fwd_bwd(prob, ws, ws_bytes, grad_loss, loss, row_loss, dH, dW, accumulate_dW, stream):
    return lib().kl_fwd_bwd(ctypes.byref(prob), ws, ws_bytes, float(grad_loss), loss, row_loss,
                            dH, dW, int(accumulate_dW), stream)


def kl_fwd_noalloc(prob, loss, lse_s, row_loss, status, stream):
    """Forward with the library's fixed static scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/chunked_kl.h)."""
    return lib().kl_fwd_noalloc(ctypes.byref(prob), loss, lse_s, row_loss, status, stream)


def kl_vp_num_chunks(prob):
    return int(lib().kl_vp_num_chunks(ctypes.byref(prob)))


def kl_vp_fwd_chunk(prob, chunk, ws, ws_bytes, row_stats, stream):
    return lib().kl_vp_fwd_chunk(ctypes.byref(prob), int(chunk), ws, ws_bytes, row_stats, stream)


def kl_vp_mid_chunk(prob, chunk, ws, ws_bytes, row_stats_all, P, rank, sums, stream):
    return lib().kl_vp_mid_chunk(ctypes.byref(prob), int(chunk), ws, ws_bytes, row_stats_all,
                                 int(P), int(rank), sums, stream)


def kl_vp_bwd_chunk(prob, chunk, ws, ws_bytes, row_stats_all, sums_all, P, rank, grad_loss, loss,
                    lse_s, row_loss, dH_part, dW, accumulate_dW, stream):
    return lib().kl_vp_bwd_chunk(ctypes.byref(prob), int(chunk), ws, ws_bytes, row_stats_all,
                                 sums_all, int(P), int(rank), float(grad_loss), loss, lse_s,
                                 row_loss, dH_part, dW, int(accumulate_dW), stream)


def kl_cast_f32(src, dst, n, dtype, stream):
    return lib().kl_cast_f32(src, dst, int(n), int(dtype), stream)


def kl_status(ws, stream):
    return lib().kl_status(ws, stream)


def kl_status_string(code):
    return _string(code)


def kl_launch_count():
    return int(lib().kl_launch_count())


def kl_profile_begin():
    check(lib().kl_profile_begin(), "kl_profile_begin")


def kl_profile_end(max_entries=64):
    arr = (KLProfileEntry * max_entries)()
    n = lib().kl_profile_end(arr, max_entries)
    if n < 0:
        raise KLError(-n, "kl_profile_end")
    return [dict(name=arr[i].name.decode(), launches=int(arr[i].launches),
                 total_ms=float(arr[i].total_ms), flops=float(arr[i].flops),
                 bytes=float(arr[i].bytes)) for i in range(min(n, max_entries))]
