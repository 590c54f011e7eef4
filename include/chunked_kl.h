/*
 * chunked_kl.h -- C ABI of the fused, chunked distillation KL loss over the
 * LM output head, for NVIDIA B200 (sm_100a).
 *
 * What the calls compute ("Efficient Knowledge Distillation for LLMs: Offline
 * Top-K Logits and a Fused Chunked KL Loss", §1 and §3; KDFlow abstract for the
 * teacher-hidden mode).  With s = H . W^T the student logits, s~ = s / T,
 * lse_s = log sum_j exp(s~_j), p_s = softmax(s~):
 *
 *   KL_TEACHER_TOPK, partial mass (teacher_lse != NULL; §3 "Offline
 *   distillation": the cached probabilities are not renormalised over K):
 *       q_i = exp(t_i / T - lse_t),  m = sum_i q_i,
 *       l_n = sum_{i in S_n} q_i (log q_i - s~_{idx_i} + lse_s)
 *           = [sum q log q] - [sum q_i s~_{idx_i}] + m * lse_s
 *       (teacher-entropy, cross and mass terms; only lse_s needs the full
 *       vocabulary).   dl_n/ds_j = (m p_s,j - q_j [j in S_n]) / T.
 *   KL_TEACHER_TOPK, renormalised (teacher_lse == NULL): q = softmax over the
 *       row's valid cached entries of t / T, m = 1, same formulas.
 *   KL_TEACHER_HIDDEN (KDFlow abstract: teacher logits recomputed from the
 *       teacher's final hidden states through a frozen teacher head):
 *       t = Ht . Wt^T,  l_n = KL(p_t || p_s),  dl_n/ds_j = (p_s,j - p_t,j) / T.
 *       With reverse_weight = beta > 0 (the KL-direction study's reverse KL and
 *       "KL mixing", thelatestinai.com/papers/2606.20005):
 *       l_n = (1 - beta) KL(p_t || p_s) + beta KL(p_s || p_t),
 *       dl_n/ds_j = [(1 - beta)(p_s,j - p_t,j) + beta p_s,j (u_j - u_bar)] / T,
 *       u = s~ - t~, u_bar = sum_j p_s,j u_j.
 *   loss = (1 / n) sum_{mask_n = 1} l_n, n = normalizer if > 0, else the number
 *       of rows with mask = 1 (0 valid rows -> loss 0, gradients 0).
 *   dS = g * dloss/ds (0 on masked rows), dH = dS . W, dW = dS^T . H.
 *   The teacher head is frozen: no gradient for Ht, Wt.
 *
 * The N x V logit tensor is never materialised (§3 "Fused chunked KL"): tokens
 * are processed in chunks of chunk_tokens rows, and the workspace holds one
 * chunk's logits, so extra memory is O(chunk_tokens * V + N).
 *
 * Conventions for every call below.
 *   - Every array argument is a DEVICE pointer owned by the caller, except
 *     kl_problem itself (host memory, read during the call only).
 *   - Row-major layouts.  H [N, d], W [V, d], Ht [N, d_t], Wt [V, d_t],
 *     topk_idx/topk_logit [N, K], mask/teacher_lse/lse/row_loss [N],
 *     dH [N, d] (same dtype as H), dW [V, d] float32.
 *   - Alignment: H, W, Ht, Wt, dH, dW must be 16-byte aligned, the workspace
 *     256-byte aligned, and d, d_t multiples of 8 (for both element types).
 *     Violations return KL_ERR_ALIGN.
 *   - stream is a cudaStream_t (passed as void*; NULL = legacy default
 *     stream).  Calls are asynchronous on it; no host synchronisation happens
 *     inside a call.  Host-detectable errors (NULL, shape, dtype, alignment,
 *     workspace size, no sm_100 device, launch failure) are returned at once
 *     and nothing is launched (or nothing further, for a launch failure).
 *   - Device-detected errors (cache index out of range or duplicated, a
 *     bounded wait that ran out) are recorded in a status word inside the
 *     workspace; read it with kl_status().  The kernels stay in bounds and
 *     finish after such an error, but the outputs are then unspecified.
 *   - The workspace must be at least kl_workspace_bytes() bytes for the same
 *     problem and entry point; its contents need not be initialised and are
 *     not meaningful between calls (except the status word).
 *   - Not re-entrant on one workspace: calls that share a workspace must be
 *     ordered (e.g. on one stream).
 */
#ifndef CHUNKED_KL_H
#define CHUNKED_KL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types of H, W, Ht, Wt, dH */
#define KL_DTYPE_BF16 0 /* bfloat16, tensor-core kind::f16, fp32 accumulation */
#define KL_DTYPE_F32 1  /* float32, tensor-core kind::tf32, fp32 accumulation  */

/* teacher modes */
#define KL_TEACHER_TOPK 0   /* offline cache: topk_idx, topk_logit (+ teacher_lse) */
#define KL_TEACHER_HIDDEN 1 /* teacher hidden states Ht through frozen head Wt     */

/* entry points, for kl_workspace_bytes */
#define KL_ENTRY_FWD 0
#define KL_ENTRY_BWD 1
#define KL_ENTRY_FWD_BWD 2

/* status codes (return values of the calls and of kl_status) */
#define KL_OK 0
#define KL_ERR_NULL 1        /* a required pointer is NULL                         */
#define KL_ERR_SHAPE 2       /* a size is out of range (N<0, d<1, V<1, K<1, ...)     */
#define KL_ERR_DTYPE 3       /* unknown dtype or teacher mode                      */
#define KL_ERR_ALIGN 4       /* pointer or row stride not 16-byte aligned          */
#define KL_ERR_WORKSPACE 5   /* ws_bytes < kl_workspace_bytes()                    */
#define KL_ERR_CUDA 6        /* a CUDA runtime call or kernel launch failed        */
#define KL_ERR_INDEX 7       /* device: cache index outside [-1, V) or duplicated  */
#define KL_ERR_TIMEOUT 8     /* device: a bounded wait inside a kernel ran out     */
#define KL_ERR_UNSUPPORTED 9 /* the current device is not sm_100 (B200-class)      */
#define KL_ERR_ARG 10        /* another bad argument (T <= 0, chunk_tokens < 0,
                                reverse_weight outside [0,1] or set in TOPK mode) */
#define KL_ERR_TOO_LARGE 11  /* kl_fwd_noalloc: one token row needs more than the
                                fixed KL_NOALLOC_SCRATCH_BYTES of scratch          */

typedef struct kl_problem {
  int64_t N;           /* tokens (rows of H); N = 0 gives loss 0 and no gradient */
  int64_t d;           /* student hidden width                                  */
  int64_t V;           /* vocabulary size (rows of W)                           */
  int32_t dtype;       /* KL_DTYPE_*: element type of H, W, Ht, Wt and dH       */
  int32_t teacher;     /* KL_TEACHER_*                                          */
  const void* H;       /* [N, d] student hidden states                          */
  const void* W;       /* [V, d] student output head (nn.Linear layout)         */
  const uint8_t* mask; /* [N] 1 = keep, 0 = ignore; NULL = keep all             */
  float T;             /* temperature, > 0, divides student and teacher logits  */
  int32_t K;           /* TOPK: cached entries per row, 1..1024                  */
  const int32_t* topk_idx;   /* TOPK: [N, K] vocabulary ids; -1 = empty slot     */
  const float* topk_logit;   /* TOPK: [N, K] teacher logits t (before / T)       */
  const float* teacher_lse;  /* TOPK: [N] log sum_j exp(t_j / T) over the full
                                vocabulary (partial mass), or NULL (renormalise) */
  int64_t d_t;               /* HIDDEN: teacher hidden width                     */
  const void* Ht;            /* HIDDEN: [N, d_t] teacher final hidden states     */
  const void* Wt;            /* HIDDEN: [V, d_t] frozen teacher output head      */
  int64_t chunk_tokens;      /* token rows per chunk; 0 = library default (4096) */
  float normalizer;          /* > 0: divide by this (e.g. a data-parallel global
                                count) instead of the number of unmasked rows    */
  float reverse_weight;      /* HIDDEN: beta in [0, 1], weight of the reverse KL
                                (0 = forward KL only); must be 0 in TOPK mode    */
  const float* T_row;        /* [N] device: temperature per token row (each > 0),
                                overriding T (the entropy-adaptive KD abstract,
                                thelatestinai.com/papers/2610.07706, adjusts the
                                temperature per token); NULL = T for every row.
                                teacher_lse must then be taken at each row's T.
                                A value <= 0 is flagged as KL_ERR_ARG in the
                                device status (kl_status).                       */
  int64_t v_begin;           /* vocabulary-parallel calls (kl_vp_*): W (and Wt)
                                hold rows [v_begin, v_begin + V) of a head with
                                V_total rows.  Must be 0 for the other calls.    */
  int64_t V_total;           /* vocabulary-parallel calls: rows of the whole
                                head; 0 or V for the other calls.  Cache ids are
                                always ids of the whole vocabulary.              */
  int32_t keep_last_chunk;   /* kl_fwd / kl_bwd only, 0 or 1.  1: kl_fwd leaves
                                the last token chunk's logits and statistics in
                                the workspace and a following kl_bwd on the same
                                workspace and the same, unchanged inputs starts
                                from them instead of recomputing that chunk's
                                projection (with N <= chunk_tokens, no recompute
                                at all).  The workspace is then the same size for
                                every entry (kl_workspace_bytes of FWD_BWD), so
                                kl_fwd's workspace grows by one chunk of logits,
                                held until kl_bwd.  Must be 0 for the other
                                calls (KL_ERR_ARG).                              */
  int32_t fuse_dlogits;      /* kl_fwd_bwd / kl_vp_* only, 0 or 1; bf16 top-K mode
                                (ignored otherwise).  1: dS is formed inside the
                                dH contraction's operand path instead of by a
                                pass over the logit chunk (§3 "Fused chunked
                                KL": logits turned into gradients on the way
                                into the gradient projections).  Same results
                                up to rounding; on B200 it measured slower than
                                the separate pass at d >= 2048 (default 0).
                                The workspace grows by one chunk of dS.  kl_fwd,
                                kl_bwd and kl_fwd_noalloc refuse it
                                (KL_ERR_ARG).                                    */
} kl_problem;

/* Bytes of workspace that entry (KL_ENTRY_*) needs for this problem, or 0 if
 * the problem is invalid.  O(chunk_tokens * V + N * 16), never O(N * V). */
size_t kl_workspace_bytes(const kl_problem* p, int entry);

/* Forward only.  Writes loss (device float scalar), lse_s [N] (log-sum-exp of
 * s~ per row, needed by kl_bwd), lse_t [N] (HIDDEN: teacher log-sum-exp; may be
 * NULL in TOPK mode) and row_loss [N] (per-row l_n, 0 on masked rows; may be
 * NULL).  Tensor work: 2 N d V (+ 2 N d_t V in HIDDEN mode). */
int kl_fwd(const kl_problem* p, void* ws, size_t ws_bytes, float* loss, float* lse_s,
           float* lse_t, float* row_loss, void* stream);

/* Backward, recomputing each chunk's logits from H and W (output-head gradient
 * checkpointing, §3 "Fused chunked KL") -- except, with keep_last_chunk, the
 * last chunk, whose logits kl_fwd left in the same workspace (it is processed
 * first).  lse_s (and lse_t in HIDDEN mode) come from kl_fwd on the same inputs.  grad_loss is a DEVICE pointer to the
 * incoming scalar gradient g.  Writes dH [N, d]; writes dW [V, d] fp32, or adds
 * to it when accumulate_dW != 0.  Tensor work: 6 N d V (+ 2 N d_t V). */
int kl_bwd(const kl_problem* p, void* ws, size_t ws_bytes, const float* lse_s,
           const float* lse_t, const float* grad_loss, void* dH, float* dW,
           int accumulate_dW, void* stream);

/* Fused forward + backward in one pass over the chunks (the logits of a chunk
 * are computed once and turned into dS in place).  grad_loss is the incoming
 * scalar gradient g by value.  Writes loss (device scalar), row_loss [N] (may
 * be NULL), dH, and dW (overwrite, or accumulate if accumulate_dW != 0).
 * Tensor work: 6 N d V (+ 2 N d_t V in HIDDEN mode). */
int kl_fwd_bwd(const kl_problem* p, void* ws, size_t ws_bytes, float grad_loss,
               float* loss, float* row_loss, void* dH, float* dW, int accumulate_dW,
               void* stream);

/* Forward-only variant for callers that cannot allocate device memory.
 *
 * No counterpart in the paper: this is a deployment convenience.  Some callers
 * cannot call cudaMalloc or hand over a workspace -- for example a plugin host
 * that passes only its input and output buffers, a runtime whose device memory
 * is planned up front and may not grow, or a code path where an allocation
 * would synchronise the device.  kl_fwd_noalloc computes what kl_fwd computes
 * (top-K mode, bf16 inputs only) without allocating anything and without a
 * workspace argument: its scratch (per-chunk tile statistics and the prepared
 * cache) lives in one fixed array of KL_NOALLOC_SCRATCH_BYTES in the library's
 * static device memory, which every GPU that loads the library holds until
 * the process exits.
 *
 * Arguments: as kl_fwd, except that row_loss [N] is required, lse_t is not
 * used, and status (device int, may be NULL) receives the device-side status
 * (KL_OK / KL_ERR_INDEX / KL_ERR_TIMEOUT) once the call's kernels finish.
 * The token chunk is the largest that fits the fixed scratch (and at most
 * chunk_tokens when that is set); results match kl_fwd up to rounding order.
 * Errors: KL_ERR_DTYPE unless bf16 + KL_TEACHER_TOPK; KL_ERR_TOO_LARGE when a
 * single token row of scratch (16 * ceil(V / 256) + 8 * K + 8 bytes, plus a
 * 256-byte header) exceeds KL_NOALLOC_SCRATCH_BYTES; the other codes as kl_fwd.
 * It calls no cudaMalloc, cudaFree or other allocating routine.  Every call
 * looks up the scratch array's device address for the current device and
 * context (cudaGetSymbolAddress, with that device current), so the address
 * stays right after a context is destroyed and created again; the first call on
 * a device may also load the library's kernels, so make it before any stream
 * capture.
 * All calls share the one array and it keeps the last call's contents (each
 * call re-initialises what it reads), so calls whose kernels overlap on the GPU
 * (different streams, or different host threads) race: order them. */
#define KL_NOALLOC_SCRATCH_BYTES (16u << 20)
int kl_fwd_noalloc(const kl_problem* p, float* loss, float* lse_s, float* row_loss,
                   int* status, void* stream);

/* ---------------------------------------------------------------- vocabulary-parallel form
 *
 * The head split by vocabulary rows over P ranks, as in tensor-parallel
 * training of the output layer (the pages' toy benchmark reports the slowest
 * tensor-parallel rank, §B "Toy Loss-Kernel Benchmark Configuration").  Rank r
 * holds W rows [v_begin, v_begin + V) of the V_total-row head (and the same
 * rows of Wt); H, mask, T / T_row and the teacher side (cache with whole-
 * vocabulary ids and teacher_lse, or Ht) are identical on every rank.  The
 * loss is exact: only the log-sum-exp over V needs every shard, and it merges
 * from per-shard values (log sum_r exp lse_r).  For every token chunk
 * k = 0 .. kl_vp_num_chunks() - 1, in order, on one workspace (size
 * kl_workspace_bytes(p, KL_ENTRY_FWD_BWD)):
 *
 *   1. kl_vp_fwd_chunk  -> row_stats [rows_k][2] of this shard
 *   2. the caller gathers all ranks' row_stats, rank-major: [P][rows_k][2]
 *      (e.g. an NCCL all-gather; 8 bytes per row per rank)
 *   (teacher-hidden mode with reverse_weight > 0 only:
 *   3a. kl_vp_mid_chunk -> sums [rows_k][2] of this shard, (A, U) below
 *   3b. the caller gathers all ranks' sums, rank-major: [P][rows_k][2])
 *   4. kl_vp_bwd_chunk  -> this rank's share of the row losses and of dH
 *      (fp32, rows of chunk k), and dW rows of its own shard
 *
 * then sums over ranks (e.g. an NCCL all-reduce) the fp32 dH partials, the
 * loss and, if wanted, row_loss: each rank's value is its share, and the sum
 * over ranks is the result.  kl_cast_f32 turns the summed fp32 dH into H's
 * dtype.  rows_k = min(C, N - k C) with C = chunk_tokens (default 4096).
 * Chunk 0 starts a pass (it resets the status word and prepares the heads);
 * the workspace carries the chunk's logits from step 1 to step 4, so no other
 * call may use it in between.  The reverse-KL gradient needs
 * u_bar = sum_j p_s,j (s~_j - t~_j) over the whole vocabulary before dS can be
 * written, hence the second exchange (A = sum_j p_t,j (t~_j - s~_j) travels with
 * it for the row loss).  Errors as kl_fwd_bwd, plus KL_ERR_ARG for v_begin < 0,
 * v_begin + V > V_total, chunk outside [0, kl_vp_num_chunks()), P < 1 or rank
 * outside [0, P). */

/* Number of token chunks of the pass (0 when N = 0), or -1 if p is invalid. */
int64_t kl_vp_num_chunks(const kl_problem* p);

/* Step 1 for chunk k: logits of the chunk over this shard (kept in ws) and the
 * rows' statistics over the shard: row_stats[i] = (lse_s over the shard, cross
 * term sum_{cached ids in the shard} q s~) in top-K mode, (lse_s, lse_t over the
 * shard) in teacher-hidden mode.  Tensor work: 2 rows_k d V (+ 2 rows_k d_t V). */
int kl_vp_fwd_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    float* row_stats, void* stream);

/* Step 3a for chunk k (KL_TEACHER_HIDDEN, else KL_ERR_ARG): from every rank's
 * step-1 output row_stats_all [P][rows_k][2], this shard's sums over its
 * columns, sums[i] = (A_r, U_r) with A_r = sum p_t (t~ - s~) and
 * U_r = sum p_s (s~ - t~), p_s and p_t the whole-vocabulary softmaxes. */
int kl_vp_mid_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    const float* row_stats_all, int P, int rank, float* sums, void* stream);

/* Step 4 for chunk k.  row_stats_all: [P][rows_k][2], every rank's step-1
 * output in rank order; sums_all: [P][rows_k][2], every rank's step-3a output
 * (required when reverse_weight > 0, ignored otherwise).  Writes lse_s [N] rows
 * of the chunk (whole-vocabulary student lse; may be NULL), row_loss [N] rows
 * of the chunk (this rank's share; may be NULL), dH_part [N, d] fp32 rows of
 * the chunk (this rank's share, dS_shard . W_shard), and dW [V, d] fp32 (this
 * shard's rows; overwritten at chunk 0 unless accumulate_dW, accumulated
 * otherwise).  After the last chunk it writes loss (device scalar, this rank's
 * share of the mean).  grad_loss is the incoming gradient g.  Tensor work:
 * 4 rows_k d V. */
int kl_vp_bwd_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    const float* row_stats_all, const float* sums_all, int P, int rank,
                    float grad_loss, float* loss, float* lse_s, float* row_loss, float* dH_part,
                    float* dW, int accumulate_dW, void* stream);

/* dst[i] = src[i] converted to dtype (KL_DTYPE_BF16: round to nearest even;
 * KL_DTYPE_F32: copy), i < n; n a multiple of 4, both 16-byte aligned. */
int kl_cast_f32(const float* src, void* dst, int64_t n, int dtype, void* stream);

/* Synchronises stream, then returns the device-side status recorded in ws
 * (KL_OK, KL_ERR_INDEX or KL_ERR_TIMEOUT), or KL_ERR_CUDA if the stream
 * reports an error.  Does not clear it; every kl_* call resets it at start. */
int kl_status(void* ws, void* stream);

/* Static English description of a status code. */
const char* kl_status_string(int code);

/* Kernel launches issued by this library since it was loaded. */
uint64_t kl_launch_count(void);

/* Per-kernel timing with CUDA events recorded on the launch stream around each
 * launch.  kl_profile_begin() clears and enables it; kl_profile_end()
 * synchronises the recorded events, disables recording and fills up to
 * max_entries entries (one per kernel kind that launched); returns the number
 * of kinds, or -KL_ERR_CUDA.  flops is the algorithmic work of all launches
 * of that kind (2 M N K for the tensor-core contractions, 0 otherwise);
 * bytes is the algorithmic HBM traffic of the memory-bound kernels. */
typedef struct kl_profile_entry {
  char name[48];
  uint64_t launches;
  double total_ms;
  double flops;
  double bytes;
} kl_profile_entry;
int kl_profile_begin(void);
int kl_profile_end(kl_profile_entry* out, int max_entries);

#ifdef __cplusplus
}
#endif

#endif /* CHUNKED_KL_H */
