// kl_api.cu -- C ABI of the fused, chunked distillation KL loss (sm_100a).
//
// Host side: argument validation, workspace planning, TMA tensor-map encoding
// and the per-chunk launch sequence ("Efficient Knowledge Distillation for
// LLMs: Offline Top-K Logits and a Fused Chunked KL Loss", §3 "Fused chunked
// KL": the output projection is fused into the loss, each logit chunk is
// transient, and backward recomputes one projection per chunk).
//
// Per chunk of C token rows (fwd_bwd, top-K):
//   prep_topk      cache -> sorted ids + teacher probabilities q, m, sum q log q
//   gemm STATS     S~ = H_c W^T / T  (tcgen05), split-V row statistics + gather,
//                  stores s~ - tile max
//   row_reduce     lse_s, row loss
//   dlogits_topk   S~ -> dS in place
//   gemm ACCUM     dH_c = dS W: wide 256 x 512 tiles, split-K fp32 parts
//   splitk_reduce  the parts summed in a fixed order -> dH_c
//   gemm ACCUM     dW (+)= dS^T H_c
// then finalize_loss (masked mean).  No host synchronisation anywhere.
// The teacher-hidden mode runs the teacher pass (fp32 t~ - tile max) and then
// the student pass, whose epilogue forms the per-tile loss sums against the
// teacher tile; hidden_sums merges them into lse_s, lse_t, the row loss and
// u_bar, and dlogits_full writes dS.  The vocabulary-parallel calls (kl_vp_*)
// split the same sequence around per-chunk exchanges.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/chunked_kl.h"
#include "kl_gemm.cuh"
#include "kl_rowops.cuh"

using namespace ckl;

namespace {

// ------------------------------------------------------------------ device
constexpr int kMaxDevices = 64;
struct DevInfo {
  int checked = 0;
  int ok = 0;
  int sms = 0;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return KL_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = sms;
    d.checked = 1;
  }
  *out = d;
  return d.ok ? KL_OK : KL_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major matrix [rows][inner] with the given row stride,
// 128-byte swizzle, zero fill outside the extents.
bool make_map(CUtensorMap* m, const void* base, int dtype, uint64_t inner, uint64_t rows,
              uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(m, dtype == KL_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
         2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output map of the GEMM epilogue: 32 x 32 boxes staged in shared memory with
// 64-byte rows (bf16, 64-byte swizzle) or 128-byte rows (fp32, 128-byte swizzle).
bool make_out_map(CUtensorMap* m, const void* base, int dtype, uint64_t inner, uint64_t rows,
                  uint64_t row_stride_bytes) {
  return make_map(m, base, dtype, inner, rows, row_stride_bytes, 32, 32,
                  dtype == KL_DTYPE_BF16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// ------------------------------------------------------------------ profiling
std::atomic<uint64_t> g_launches{0};

struct ProfKind {
  std::string name;
  uint64_t launches = 0;
  double flops = 0, bytes = 0;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::deque<ProfKind> g_prof;  // deque: LaunchScope keeps pointers to its entries
std::vector<cudaEvent_t> g_ev_pool;

cudaEvent_t pool_event() {
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct LaunchScope {
  cudaStream_t st;
  ProfKind* kind = nullptr;
  cudaEvent_t e0 = nullptr;
  LaunchScope(const char* name, cudaStream_t s, double flops, double bytes) : st(s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return;
    for (auto& k : g_prof)
      if (k.name == name) kind = &k;
    if (kind == nullptr) {
      g_prof.push_back(ProfKind());
      kind = &g_prof.back();
      kind->name = name;
    }
    kind->launches++;
    kind->flops += flops;
    kind->bytes += bytes;
    e0 = pool_event();
    cudaEventRecord(e0, st);
  }
  ~LaunchScope() {
    if (kind == nullptr) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t e1 = pool_event();
    cudaEventRecord(e1, st);
    kind->ev.emplace_back(e0, e1);
  }
};

long long spin_limit() {
  static long long lim = [] {
    const char* s = getenv("KL_SPIN_LIMIT");
    long long v = s ? atoll(s) : 0;
    return v > 0 ? v : 4000000000LL;  // ~2 s at the B200 boost clock
  }();
  return lim;
}

#define KL_TRY(x)                 \
  do {                            \
    const int _e = (x);           \
    if (_e != KL_OK) return _e;   \
  } while (0)

// ------------------------------------------------------------------ planning
constexpr int64_t kDefaultChunk = 4096;
constexpr int kMaxK = 1024;

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  int eb = 2;          // element bytes
  int64_t C = 0;       // chunk rows
  int64_t Vp = 0;      // padded logit-buffer row length (multiple of 8)
  int tiles_v = 0;     // 256-column tiles over V
  bool hidden = false;
  // workspace offsets (bytes)
  size_t off_sbuf = 0, off_tbuf = 0, off_ps = 0, off_pt = 0, off_sidx = 0, off_sq = 0,
         off_rinfo = 0, off_lse_s = 0, off_lse_t = 0, off_rl = 0, total = 0;
  // fp32 (tf32) path only: tf32-rounded operand copies (heads W, Wt; the
  // current chunk of H or Ht) and K-major copies W^T [d][Vp], dS^T [V][Cp],
  // H_c^T [d][Cp] for the gradient contractions.
  int64_t Cp = 0;
  // fuse_dlogits (bf16 top-K): the logits pass stores exponentials, the dH
  // contraction forms dS from them in shared memory and stores it for dW
  bool xf = false;
  int64_t Cx = 0;          // (xf) row stride of the transposed dS scales: C rounded up to 64
  size_t off_xsc = 0;      // (xf) dS scales [tiles_v][Cx] fp32
  size_t off_dsbuf = 0;    // (xf) dS chunk [C][Vp] bf16
  size_t off_ubar = 0;     // (hidden) u_bar per chunk row
  int ksplit_dh = 1;       // K-parts of the dH contraction (fp32 partials + reduce)
  size_t off_dhp = 0;      // dH partials [ksplit_dh][C][d] fp32
  size_t off_wr = 0, off_wtr = 0, off_xr = 0, off_wT = 0, off_sT = 0, off_hT = 0;
};

// Sizes, dtypes and scalar arguments (no pointers).
// Number of K-parts for a contraction with `tiles` output tiles and `num_kb`
// K-blocks on `units` CTA pairs: the smallest split (at most 8, each part at
// least 32 K-blocks) whose last wave is fullest.  Every part is non-empty.
int choose_ksplit(int64_t tiles, int64_t num_kb, int64_t units) {
  int best = 1;
  double best_eff = 0;
  for (int s = 1; s <= 8; ++s) {
    if (num_kb / s < 32 && s > 1) break;
    const int64_t kbs = cdiv(num_kb, s);
    if ((s - 1) * kbs >= num_kb) continue;  // an empty part
    const int64_t u = tiles * s;
    const double eff = static_cast<double>(u) / (cdiv(u, units) * units);
    if (eff > best_eff + 0.01) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

// dH (bf16) runs on wide 256 x 512 pair tiles: its work units are long (a
// K-part of the vocabulary), so the single accumulator's unhidden epilogue
// costs little, and sharing each A stage between two N halves cuts the operand
// bytes a CTA pulls from L2 by a quarter.
constexpr int kDhWide = 1;
constexpr int kDhTileN = kDhWide ? 2 * kBN : kBN;

// CTA pairs available for one contraction (the workspace plan must not depend
// on the device, so this is the B200's 148 SMs / 2).
int64_t max_units_hint() { return 74; }

int validate_shape(const kl_problem* p) {
  if (p == nullptr) return KL_ERR_NULL;
  if (p->dtype != KL_DTYPE_BF16 && p->dtype != KL_DTYPE_F32) return KL_ERR_DTYPE;
  if (p->teacher != KL_TEACHER_TOPK && p->teacher != KL_TEACHER_HIDDEN) return KL_ERR_DTYPE;
  if (p->N < 0 || p->d < 1 || p->V < 1 || p->N > (int64_t(1) << 31) - 1 ||
      p->V > (int64_t(1) << 31) - 512 || p->d > (int64_t(1) << 20))
    return KL_ERR_SHAPE;
  if (!(p->T > 0.f) || !(p->T < INFINITY) || p->chunk_tokens < 0 || !(p->normalizer >= 0.f))
    return KL_ERR_ARG;
  if (!(p->reverse_weight >= 0.f && p->reverse_weight <= 1.f) ||
      (p->reverse_weight > 0.f && p->teacher != KL_TEACHER_HIDDEN))
    return KL_ERR_ARG;
  if (p->keep_last_chunk != 0 && p->keep_last_chunk != 1) return KL_ERR_ARG;
  if (p->fuse_dlogits != 0 && p->fuse_dlogits != 1) return KL_ERR_ARG;
  if (p->v_begin < 0 || p->V_total < 0 || p->V_total > (int64_t(1) << 31) - 512 ||
      (p->V_total > 0 && p->v_begin + p->V > p->V_total) || (p->V_total == 0 && p->v_begin != 0))
    return KL_ERR_ARG;
  if (p->d % 8 != 0) return KL_ERR_ALIGN;
  if (p->teacher == KL_TEACHER_TOPK) {
    if (p->K < 1 || p->K > kMaxK) return KL_ERR_SHAPE;
  } else {
    if (p->d_t < 1 || p->d_t > (int64_t(1) << 20)) return KL_ERR_SHAPE;
    if (p->d_t % 8 != 0) return KL_ERR_ALIGN;
  }
  return KL_OK;
}

int validate(const kl_problem* p) {
  KL_TRY(validate_shape(p));
  if (p->N > 0) {
    if (p->H == nullptr || p->W == nullptr) return KL_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(p->H) | reinterpret_cast<uintptr_t>(p->W)) & 15)
      return KL_ERR_ALIGN;
    if (p->teacher == KL_TEACHER_TOPK) {
      if (p->topk_idx == nullptr || p->topk_logit == nullptr) return KL_ERR_NULL;
    } else {
      if (p->Ht == nullptr || p->Wt == nullptr) return KL_ERR_NULL;
      if ((reinterpret_cast<uintptr_t>(p->Ht) | reinterpret_cast<uintptr_t>(p->Wt)) & 15)
        return KL_ERR_ALIGN;
    }
  }
  return KL_OK;
}

// Rows of the whole head (the vocabulary the cache ids index).
int64_t vocab_total(const kl_problem* p) { return p->V_total > 0 ? p->V_total : p->V; }
// The problem covers the whole head (every call except kl_vp_*).
bool whole_head(const kl_problem* p) { return p->v_begin == 0 && vocab_total(p) == p->V; }

Plan make_plan(const kl_problem* p, int entry) {
  // a kept chunk passes from kl_fwd to kl_bwd in one layout: the fused pass's
  if (p->keep_last_chunk) entry = KL_ENTRY_FWD_BWD;
  Plan pl;
  pl.eb = p->dtype == KL_DTYPE_BF16 ? 2 : 4;
  pl.hidden = p->teacher == KL_TEACHER_HIDDEN;
  const int64_t chunk = p->chunk_tokens > 0 ? p->chunk_tokens : kDefaultChunk;
  pl.C = p->N < chunk ? p->N : chunk;
  if (pl.C < 1) pl.C = 1;
  pl.Vp = cdiv(p->V, 8) * 8;
  pl.tiles_v = static_cast<int>(cdiv(p->V, kBN));
  pl.xf = p->fuse_dlogits && pl.eb == 2 && !pl.hidden;
  // student logits / dS chunk: wherever dS is formed (not the forward alone)
  const bool need_sbuf = entry != KL_ENTRY_FWD;
  // tile statistics: every pass that computes them (the top-K backward forms
  // dS in its recompute epilogue from the known lse and needs none)
  const bool need_stats = entry != KL_ENTRY_BWD || pl.hidden;
  size_t off = 256;  // Scalars
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes);
    return o;
  };
  const size_t buf = static_cast<size_t>(pl.C) * pl.Vp * pl.eb;
  if (need_sbuf) pl.off_sbuf = take(buf);
  // teacher logits chunk, fp32: the student pass forms the loss sums from it
  if (pl.hidden) pl.off_tbuf = take(static_cast<size_t>(pl.C) * pl.Vp * 4);
  if (need_stats) pl.off_ps = take(static_cast<size_t>(pl.C) * pl.tiles_v * sizeof(float4));
  if (need_stats && pl.hidden)
    pl.off_pt = take(static_cast<size_t>(pl.C) * pl.tiles_v * sizeof(float4));
  if (pl.hidden && entry != KL_ENTRY_FWD) pl.off_ubar = take(static_cast<size_t>(pl.C) * 4);
  if (pl.xf && entry == KL_ENTRY_FWD_BWD) {
    pl.Cx = cdiv(pl.C, 64) * 64;
    pl.off_xsc = take(static_cast<size_t>(pl.tiles_v) * pl.Cx * 4);
    pl.off_dsbuf = take(buf);  // dS chunk, formed by the dH contraction for dW
  }
  if (!pl.hidden) {
    pl.off_sidx = take(static_cast<size_t>(pl.C) * p->K * 4);
    pl.off_sq = take(static_cast<size_t>(pl.C) * p->K * 4);
    pl.off_rinfo = take(static_cast<size_t>(pl.C) * sizeof(float2));
  }
  const size_t nrow = static_cast<size_t>(p->N > 0 ? p->N : 1) * 4;
  if (entry == KL_ENTRY_FWD_BWD) {
    pl.off_lse_s = take(nrow);
    if (pl.hidden) pl.off_lse_t = take(nrow);
  }
  if (entry != KL_ENTRY_BWD) pl.off_rl = take(nrow);
  if (pl.eb == 2 && entry != KL_ENTRY_FWD) {
    pl.ksplit_dh = choose_ksplit(cdiv(pl.C, 2 * kBM) * cdiv(p->d, kDhTileN), cdiv(p->V, 64),
                                 max_units_hint());
    if (pl.ksplit_dh > 1)
      pl.off_dhp = take(static_cast<size_t>(pl.ksplit_dh) * cdiv(pl.C, 2 * kBM) * 2 * kBM *
                        p->d * 4);
  }
  if (pl.eb == 4) {
    const int64_t dmax = (pl.hidden && p->d_t > p->d) ? p->d_t : p->d;
    pl.off_wr = take(static_cast<size_t>(p->V) * p->d * 4);
    if (pl.hidden) pl.off_wtr = take(static_cast<size_t>(p->V) * p->d_t * 4);
    pl.off_xr = take(static_cast<size_t>(pl.C) * dmax * 4);
  }
  if (pl.eb == 4 && entry != KL_ENTRY_FWD) {
    pl.Cp = cdiv(pl.C, 4) * 4;
    pl.off_wT = take(static_cast<size_t>(p->d) * pl.Vp * 4);
    pl.off_sT = take(static_cast<size_t>(p->V) * pl.Cp * 4);
    pl.off_hT = take(static_cast<size_t>(p->d) * pl.Cp * 4);
  }
  pl.total = off;
  return pl;
}

// ------------------------------------------------------------------ launches
template <typename Elem, int A_MN, int B_MN, int EPI, int PAIR = 0, int WIDE = 0, int XF = 0,
          int EG = 1>
int launch_gemm(const char* name, cudaStream_t st, int sms, const CUtensorMap& ma,
                const CUtensorMap& mb, const CUtensorMap& mc, GemmParams gp, double flops,
                const CUtensorMap* md = nullptr) {
  auto kern = gemm_tc_kernel<Elem, A_MN, B_MN, EPI, PAIR, WIDE, XF, EG>;
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev].load()) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
        cudaSuccess)
      return KL_ERR_CUDA;
    attr_set[dev].store(true);
  }
  const int tiles = gp.tiles_m * gp.tiles_n * gp.ksplit;  // work units
  const int units = PAIR ? sms / 2 : sms;  // CTA pairs or CTAs, one CTA per SM
  const int grid = (tiles < units ? tiles : units) * (PAIR ? 2 : 1);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((XF || EG == 2) ? kGemmThreadsXf : kGemmThreads);
  cfg.dynamicSmemBytes = kGemmSmemBytes;
  cfg.stream = st;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e;
  {
    LaunchScope ls(name, st, flops, 0);
    e = cudaLaunchKernelEx(&cfg, kern, ma, mb, mc, md != nullptr ? *md : mc, gp);
  }
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? KL_OK : KL_ERR_CUDA;
}

#define KL_LAUNCHED() (cudaGetLastError() == cudaSuccess ? KL_OK : KL_ERR_CUDA)

struct Ctx {
  const kl_problem* p;
  Plan pl;
  uint8_t* ws;
  Scalars* sc;
  cudaStream_t st;
  int sms;
  float invT;
};

int launch_round(Ctx& c, const float* src, int64_t ld_src, float* dst, int64_t ld_dst,
                 int64_t rows, int64_t cols) {
  LaunchScope ls("round_tf32", c.st, 0, 8.0 * rows * cols);
  round_tf32_kernel<<<static_cast<unsigned>(c.sms * 8), 256, 0, c.st>>>(src, ld_src, dst, ld_dst,
                                                                       rows, cols);
  return cudaGetLastError() == cudaSuccess ? KL_OK : KL_ERR_CUDA;
}

// Heads as the logits contraction reads them (tf32-rounded copies for fp32).
const void* head_W(Ctx& c) {
  return c.pl.eb == 4 ? static_cast<const void*>(c.ws + c.pl.off_wr) : c.p->W;
}
const void* head_Wt(Ctx& c) {
  return c.pl.eb == 4 ? static_cast<const void*>(c.ws + c.pl.off_wtr) : c.p->Wt;
}
int prepare_heads(Ctx& c) {
  if (c.pl.eb != 4) return KL_OK;
  const kl_problem* p = c.p;
  KL_TRY(launch_round(c, static_cast<const float*>(p->W), p->d,
                      reinterpret_cast<float*>(c.ws + c.pl.off_wr), p->d, p->V, p->d));
  if (c.pl.hidden)
    KL_TRY(launch_round(c, static_cast<const float*>(p->Wt), p->d_t,
                        reinterpret_cast<float*>(c.ws + c.pl.off_wtr), p->d_t, p->V, p->d_t));
  return KL_OK;
}

// Logits pass over one chunk: S~ = X_c . Wh^T / T with the tile statistics in
// `partials`; out != nullptr: s~ - tile max stored into `out` (fp32 when
// out_f32, else the input type), or with exp_store the bf16 exponentials
// 2^(s~ log2 e - tile max) (the fused-dS path).  tbuf / tpart: the teacher
// pass's stored tile and statistics (student pass of the teacher-hidden mode:
// the tile sums A and U go to partials .z / .w).
template <typename Elem>
int gemm_logits(Ctx& c, const void* X, int64_t dx, const void* Wh, int64_t c0, int64_t Cn,
                void* out, bool out_f32, float4* partials, const int* sidx,
                const float* sq, int ktop, const char* name, const float* tbuf = nullptr,
                const float4* tpart = nullptr, bool exp_store = false) {
  const kl_problem* p = c.p;
  constexpr int kBKe = kRowBytes / sizeof(Elem);
  CUtensorMap ma, mb;
  const uint8_t* xc = static_cast<const uint8_t*>(X) + c0 * dx * sizeof(Elem);
  if (sizeof(Elem) == 4) {  // tf32: round the chunk of hidden states first
    float* xr = reinterpret_cast<float*>(c.ws + c.pl.off_xr);
    KL_TRY(launch_round(c, reinterpret_cast<const float*>(xc), dx, xr, dx, Cn, dx));
    xc = reinterpret_cast<const uint8_t*>(xr);
  }
  CUtensorMap mc;
  if (!make_map(&ma, xc, p->dtype, dx, Cn, dx * sizeof(Elem), kBKe, kBM) ||
      !make_map(&mb, Wh, p->dtype, dx, p->V, dx * sizeof(Elem), kBKe, kBN / 2))
    return KL_ERR_CUDA;
  if (out != nullptr) {
    out_f32 = out_f32 && !exp_store;
    if (!make_out_map(&mc, out, out_f32 ? KL_DTYPE_F32 : p->dtype, p->V, Cn,
                      c.pl.Vp * (out_f32 ? 4 : sizeof(Elem))))
      return KL_ERR_CUDA;
  } else {
    mc = mb;  // statistics only: the output map is not used
  }
  GemmParams gp{};
  gp.tiles_m = static_cast<int>(cdiv(Cn, 2 * kBM));
  gp.tiles_n = c.pl.tiles_v;
  gp.num_kb = static_cast<int>(cdiv(dx, kBKe));
  gp.m_fastest = 1;
  gp.store = out == nullptr ? STORE_NONE : exp_store ? STORE_EXP : STORE_SHIFTED;
  gp.out_f32 = out_f32 ? 1 : 0;
  gp.rows_valid = static_cast<int>(Cn);
  gp.cols_valid = static_cast<int>(p->V);
  gp.scale = c.invT;
  gp.T_row = p->T_row ? p->T_row + c0 : nullptr;
  gp.partials = partials;
  gp.sidx = sidx;
  gp.sq = sq;
  gp.ktop = ktop;
  gp.tbuf = tbuf;
  gp.tld = c.pl.Vp;
  gp.tpart = tpart;
  gp.status = &c.sc->status;
  gp.spin_limit = spin_limit();
  if constexpr (sizeof(Elem) == 2) {
    // The student pass of the teacher-hidden mode reads the fp32 teacher tile
    // and forms two exponentials per element: its epilogue outlasts a unit's
    // MMAs, so two epilogue groups take alternate units.
    if (tbuf != nullptr)
      return launch_gemm<Elem, 0, 0, EPI_STATS, 1, 0, 0, 2>(name, c.st, c.sms, ma, mb, mc, gp,
                                                            2.0 * Cn * p->V * dx);
  }
  return launch_gemm<Elem, 0, 0, EPI_STATS, 1>(name, c.st, c.sms, ma, mb, mc, gp,
                                               2.0 * Cn * p->V * dx);
}

int launch_transpose(Ctx& c, const float* src, int64_t ld_src, float* dst, int64_t ld_dst,
                     int64_t rows, int64_t cols) {
  LaunchScope ls("transpose_f32", c.st, 0, 8.0 * rows * cols);
  dim3 grid(static_cast<unsigned>(cdiv(cols, 32)), static_cast<unsigned>(cdiv(rows, 32)));
  transpose_f32_kernel<<<grid, dim3(32, 8), 0, c.st>>>(src, ld_src, dst, ld_dst,
                                                       static_cast<int>(rows),
                                                       static_cast<int>(cols));
  return cudaGetLastError() == cudaSuccess ? KL_OK : KL_ERR_CUDA;
}

// fp32 inputs: both gradient contractions with K-major tf32 operands only.
int gemm_grads_f32(Ctx& c, float* dS, int64_t c0, int64_t Cn, void* dH, float* dW, int beta) {
  const kl_problem* p = c.p;
  const int64_t d = p->d, V = p->V, Cp = c.pl.Cp;
  float* sT = reinterpret_cast<float*>(c.ws + c.pl.off_sT);
  float* hT = reinterpret_cast<float*>(c.ws + c.pl.off_hT);
  const float* wT = reinterpret_cast<const float*>(c.ws + c.pl.off_wT);
  const float* hc = static_cast<const float*>(p->H) + c0 * d;
  KL_TRY(launch_transpose(c, dS, c.pl.Vp, sT, Cp, Cn, V));
  KL_TRY(launch_transpose(c, hc, d, hT, Cp, Cn, d));
  {
    CUtensorMap ma, mb, mc;
    if (!make_map(&ma, dS, p->dtype, V, Cn, c.pl.Vp * 4, 32, kBM) ||
        !make_map(&mb, wT, p->dtype, V, d, c.pl.Vp * 4, 32, kBN / 2) ||
        !make_out_map(&mc, static_cast<float*>(dH) + c0 * d, KL_DTYPE_F32, d, Cn, d * 4))
      return KL_ERR_CUDA;
    GemmParams gp{};
    gp.tiles_m = static_cast<int>(cdiv(Cn, 2 * kBM));
    gp.tiles_n = static_cast<int>(cdiv(d, kBN));
    gp.num_kb = static_cast<int>(cdiv(V, 32));
    gp.m_fastest = 1;
    gp.rows_valid = static_cast<int>(Cn);
    gp.cols_valid = static_cast<int>(d);
    gp.status = &c.sc->status;
    gp.spin_limit = spin_limit();
    KL_TRY((launch_gemm<float, 0, 0, EPI_STORE, 1>("gemm_dH", c.st, c.sms, ma, mb, mc, gp,
                                                   2.0 * Cn * V * d)));
  }
  {
    CUtensorMap ma, mb, mc;
    if (!make_map(&ma, sT, p->dtype, Cn, V, Cp * 4, 32, kBM) ||
        !make_map(&mb, hT, p->dtype, Cn, d, Cp * 4, 32, kBN / 2) ||
        !make_out_map(&mc, dW, KL_DTYPE_F32, d, V, d * 4))
      return KL_ERR_CUDA;
    GemmParams gp{};
    gp.tiles_m = static_cast<int>(cdiv(V, 2 * kBM));
    gp.tiles_n = static_cast<int>(cdiv(d, kBN));
    gp.num_kb = static_cast<int>(cdiv(Cn, 32));
    gp.m_fastest = 0;
    gp.rows_valid = static_cast<int>(V);
    gp.cols_valid = static_cast<int>(d);
    gp.beta = beta;
    gp.status = &c.sc->status;
    gp.spin_limit = spin_limit();
    KL_TRY((launch_gemm<float, 0, 0, EPI_ACCUM, 1>("gemm_dW", c.st, c.sms, ma, mb, mc, gp,
                                                   2.0 * Cn * V * d)));
  }
  return KL_OK;
}

// Backward with known lse (split path, top-K mode): the recomputed logits tile
// becomes dS in the GEMM epilogue and is stored to the chunk buffer.
template <typename Elem>
int gemm_dlogits(Ctx& c, Elem* S, int64_t c0, int64_t Cn, const float* lse_s, const float* g_dev,
                 float g_host) {
  const kl_problem* p = c.p;
  constexpr int kBKe = kRowBytes / sizeof(Elem);
  const int64_t dx = p->d;
  CUtensorMap ma, mb, mc;
  const uint8_t* xc = static_cast<const uint8_t*>(p->H) + c0 * dx * sizeof(Elem);
  if (sizeof(Elem) == 4) {  // tf32: round the chunk of hidden states first
    float* xr = reinterpret_cast<float*>(c.ws + c.pl.off_xr);
    KL_TRY(launch_round(c, reinterpret_cast<const float*>(xc), dx, xr, dx, Cn, dx));
    xc = reinterpret_cast<const uint8_t*>(xr);
  }
  if (!make_map(&ma, xc, p->dtype, dx, Cn, dx * sizeof(Elem), kBKe, kBM) ||
      !make_map(&mb, head_W(c), p->dtype, dx, p->V, dx * sizeof(Elem), kBKe, kBN / 2) ||
      !make_out_map(&mc, S, p->dtype, p->V, Cn, c.pl.Vp * sizeof(Elem)))
    return KL_ERR_CUDA;
  GemmParams gp{};
  gp.tiles_m = static_cast<int>(cdiv(Cn, 2 * kBM));
  gp.tiles_n = c.pl.tiles_v;
  gp.num_kb = static_cast<int>(cdiv(dx, kBKe));
  gp.m_fastest = 1;
  gp.store = 1;
  gp.rows_valid = static_cast<int>(Cn);
  gp.cols_valid = static_cast<int>(p->V);
  gp.scale = c.invT;
  gp.T_row = p->T_row ? p->T_row + c0 : nullptr;
  gp.sidx = reinterpret_cast<const int*>(c.ws + c.pl.off_sidx);
  gp.sq = reinterpret_cast<const float*>(c.ws + c.pl.off_sq);
  gp.ktop = p->K;
  gp.lse = lse_s + c0;
  gp.rowinfo = reinterpret_cast<const float2*>(c.ws + c.pl.off_rinfo);
  gp.mask = p->mask ? p->mask + c0 : nullptr;
  gp.norm = &c.sc->norm;
  gp.g_dev = g_dev;
  gp.g_host = g_host;
  gp.status = &c.sc->status;
  gp.spin_limit = spin_limit();
  return launch_gemm<Elem, 0, 0, EPI_DLOGITS, 1>("gemm_dlogits", c.st, c.sms, ma, mb, mc, gp,
                                                 2.0 * Cn * p->V * dx);
}

// dH_c = dS . W and dW (+)= dS^T . H_c for chunk rows [c0, c0 + Cn) from the
// chunk buffer dS.  dH_f32: write dH as fp32 (a vocabulary shard's partial sum)
// whatever Elem is.  XF = 1: the buffer holds the logits pass's exponentials,
// patched at the cached columns (xf_patch_kernel); the dH contraction forms
// dS = scale * e in shared memory with the per-(tile, row) scales xf_sc and
// stores it to the workspace's dS chunk, which the dW contraction reads.
template <typename Elem, int XF>
int gemm_grads_bf16(Ctx& c, Elem* dS, int64_t c0, int64_t Cn, void* dH, float* dW, int beta,
                    bool dH_f32, const float* xf_sc) {
  const kl_problem* p = c.p;
  constexpr int kBKe = kRowBytes / sizeof(Elem);
  constexpr int kMNe = kRowBytes / sizeof(Elem);
  const int64_t d = p->d;
  const uint64_t ldS = c.pl.Vp * sizeof(Elem);
  Elem* dS_formed = XF ? reinterpret_cast<Elem*>(c.ws + c.pl.off_dsbuf) : dS;
  CUtensorMap md;  // XF: the dS chunk written by the dH contraction, 64 x 32 boxes
  if (XF && !make_map(&md, dS_formed, p->dtype, p->V, Cn, ldS, kBKe, 32)) return KL_ERR_CUDA;
  auto set_xf = [&](GemmParams& gp) {
    if (!XF) return;
    gp.xf_sc = xf_sc;
    gp.xf_ld = c.pl.Cx;
    gp.xf_rows = static_cast<int>(Cn);
    gp.xf_store = 1;
  };
  // dH_c = dS . W : A = dS [Cn, V] K-major, B = W as [d, V] MN-major.  When the
  // output has too few tiles to fill the GPU, V is split into ksplit parts whose
  // fp32 partial products are summed in a fixed order afterwards.
  {
    CUtensorMap ma, mb;
    if (!make_map(&ma, dS, p->dtype, p->V, Cn, ldS, kBKe, kBM) ||
        !make_map(&mb, p->W, p->dtype, d, p->V, d * sizeof(Elem), kMNe, kBKe))
      return KL_ERR_CUDA;
    GemmParams gp{};
    gp.tiles_m = static_cast<int>(cdiv(Cn, 2 * kBM));
    gp.tiles_n = static_cast<int>(cdiv(d, kDhTileN));
    gp.num_kb = static_cast<int>(cdiv(p->V, kBKe));
    gp.m_fastest = 1;
    gp.rows_valid = static_cast<int>(Cn);
    gp.cols_valid = static_cast<int>(d);
    gp.status = &c.sc->status;
    gp.spin_limit = spin_limit();
    set_xf(gp);
    int ks = choose_ksplit(static_cast<int64_t>(gp.tiles_m) * gp.tiles_n, gp.num_kb, c.sms / 2);
    if (ks > c.pl.ksplit_dh) ks = c.pl.ksplit_dh;
    if (ks > 1) {
      float* part = reinterpret_cast<float*>(c.ws + c.pl.off_dhp);
      // Each K-part owns a slice padded to whole 256-row tiles: output boxes
      // that overhang the chunk's last row land in the part's own padding,
      // never in the next part's rows.
      const int64_t rows_pad = cdiv(Cn, 2 * kBM) * 2 * kBM;
      gp.ksplit = ks;
      gp.split_rows = static_cast<int>(rows_pad);
      gp.beta = 0;
      CUtensorMap mc;
      if (!make_out_map(&mc, part, KL_DTYPE_F32, d, static_cast<uint64_t>(ks) * rows_pad, d * 4))
        return KL_ERR_CUDA;
      KL_TRY((launch_gemm<Elem, 0, 1, EPI_ACCUM, 1, kDhWide, XF>("gemm_dH", c.st, c.sms, ma, mb,
                                                                 mc, gp, 2.0 * Cn * p->V * d,
                                                                 XF ? &md : nullptr)));
      LaunchScope ls("splitk_reduce", c.st, 0,
                     (4.0 * ks + (dH_f32 ? 4.0 : sizeof(Elem))) * Cn * d);
      if (dH_f32)
        splitk_reduce_kernel<float><<<static_cast<unsigned>(c.sms * 8), 256, 0, c.st>>>(
            part, ks, rows_pad * d, static_cast<float*>(dH) + c0 * d, Cn * d);
      else
        splitk_reduce_kernel<Elem><<<static_cast<unsigned>(c.sms * 8), 256, 0, c.st>>>(
            part, ks, rows_pad * d, static_cast<Elem*>(dH) + c0 * d, Cn * d);
      KL_TRY(cudaGetLastError() == cudaSuccess ? KL_OK : KL_ERR_CUDA);
    } else if (dH_f32) {
      // fp32 store straight into the chunk's rows (boxes past row Cn are clipped)
      gp.beta = 0;
      CUtensorMap mc;
      if (!make_out_map(&mc, static_cast<float*>(dH) + c0 * d, KL_DTYPE_F32, d, Cn, d * 4))
        return KL_ERR_CUDA;
      KL_TRY((launch_gemm<Elem, 0, 1, EPI_ACCUM, 1, kDhWide, XF>("gemm_dH", c.st, c.sms, ma, mb,
                                                                 mc, gp, 2.0 * Cn * p->V * d,
                                                                 XF ? &md : nullptr)));
    } else {
      CUtensorMap mc;
      if (!make_out_map(&mc, static_cast<uint8_t*>(dH) + c0 * d * sizeof(Elem), p->dtype, d, Cn,
                        d * sizeof(Elem)))
        return KL_ERR_CUDA;
      KL_TRY((launch_gemm<Elem, 0, 1, EPI_STORE, 1, kDhWide, XF>("gemm_dH", c.st, c.sms, ma, mb,
                                                                 mc, gp, 2.0 * Cn * p->V * d,
                                                                 XF ? &md : nullptr)));
    }
  }
  // dW (+)= dS^T . H_c : A = dS^T [V, Cn] MN-major, B = H_c as [d, Cn] MN-major.
  {
    CUtensorMap ma, mb, mc;
    const uint8_t* hc = static_cast<const uint8_t*>(p->H) + c0 * d * sizeof(Elem);
    if (!make_map(&ma, dS_formed, p->dtype, p->V, Cn, ldS, kMNe, kBKe) ||
        !make_map(&mb, hc, p->dtype, d, Cn, d * sizeof(Elem), kMNe, kBKe) ||
        !make_out_map(&mc, dW, KL_DTYPE_F32, d, p->V, d * 4))
      return KL_ERR_CUDA;
    GemmParams gp{};
    gp.tiles_m = static_cast<int>(cdiv(p->V, 2 * kBM));
    gp.tiles_n = static_cast<int>(cdiv(d, kBN));
    gp.num_kb = static_cast<int>(cdiv(Cn, kBKe));
    gp.m_fastest = 0;
    gp.rows_valid = static_cast<int>(p->V);
    gp.cols_valid = static_cast<int>(d);
    gp.beta = beta;
    gp.status = &c.sc->status;
    gp.spin_limit = spin_limit();
    KL_TRY((launch_gemm<Elem, 1, 1, EPI_ACCUM, 1>("gemm_dW", c.st, c.sms, ma, mb, mc, gp,
                                                  2.0 * Cn * p->V * d)));
  }
  return KL_OK;
}

// dH_f32: write dH as fp32 (a vocabulary shard's partial sum) whatever Elem is.
// xf_sc != nullptr: the fused-dS path (bf16), dS formed in dH's operand path.
template <typename Elem>
int gemm_grads(Ctx& c, Elem* dS, int64_t c0, int64_t Cn, void* dH, float* dW, int beta,
               bool dH_f32 = false, const float* xf_sc = nullptr) {
  if (sizeof(Elem) == 4)
    return gemm_grads_f32(c, reinterpret_cast<float*>(dS), c0, Cn, dH, dW, beta);
  using B = __nv_bfloat16;
  B* b = reinterpret_cast<B*>(dS);
  return xf_sc != nullptr ? gemm_grads_bf16<B, 1>(c, b, c0, Cn, dH, dW, beta, dH_f32, xf_sc)
                          : gemm_grads_bf16<B, 0>(c, b, c0, Cn, dH, dW, beta, dH_f32, nullptr);
}

int launch_count_valid(Ctx& c) {
  LaunchScope ls("count_valid", c.st, 0, static_cast<double>(c.p->mask ? c.p->N : 0));
  count_valid_kernel<<<1, 1024, 0, c.st>>>(c.p->mask, c.p->N, c.p->normalizer, c.p->T_row, c.sc);
  return KL_LAUNCHED();
}

int launch_prep(Ctx& c, int64_t c0, int64_t Cn) {
  const kl_problem* p = c.p;
  const int K = p->K;
  const int rows_per_block = 4;
  const size_t smem = static_cast<size_t>(rows_per_block) * 3 * K * 4;
  int* sidx = reinterpret_cast<int*>(c.ws + c.pl.off_sidx);
  float* sq = reinterpret_cast<float*>(c.ws + c.pl.off_sq);
  float2* rinfo = reinterpret_cast<float2*>(c.ws + c.pl.off_rinfo);
  static std::atomic<bool> attr[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev].load()) {
    cudaFuncSetAttribute(prep_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         rows_per_block * 3 * kMaxK * 4);
    attr[dev].store(true);
  }
  LaunchScope ls("prep_topk", c.st, 0, static_cast<double>(Cn) * K * 16 + Cn * 12);
  prep_topk_kernel<<<static_cast<unsigned>(cdiv(Cn, rows_per_block)), 32 * rows_per_block, smem,
                     c.st>>>(p->topk_idx + c0 * K, p->topk_logit + c0 * K,
                             p->teacher_lse ? p->teacher_lse + c0 : nullptr, c.invT,
                             p->T_row ? p->T_row + c0 : nullptr,
                             static_cast<int>(vocab_total(p)), K, static_cast<int>(Cn), sidx, sq,
                             rinfo, c.sc, static_cast<int>(p->v_begin), static_cast<int>(p->V));
  return KL_LAUNCHED();
}

int launch_row_reduce(Ctx& c, const float4* partials, int64_t c0, int64_t Cn, bool with_loss,
                      float* lse_out, float* row_loss) {
  const kl_problem* p = c.p;
  const float2* rinfo =
      with_loss ? reinterpret_cast<const float2*>(c.ws + c.pl.off_rinfo) : nullptr;
  LaunchScope ls("row_reduce", c.st, 0, static_cast<double>(Cn) * c.pl.tiles_v * 16);
  row_reduce_kernel<<<static_cast<unsigned>(cdiv(Cn, 8)), 256, 0, c.st>>>(
      partials, c.pl.tiles_v, static_cast<int>(Cn), p->mask ? p->mask + c0 : nullptr, rinfo,
      lse_out + c0, row_loss ? row_loss + c0 : nullptr, 1, nullptr);
  return KL_LAUNCHED();
}

// A vocabulary shard's row statistics, interleaved pairs: lse -> out[2 i + slot],
// and in top-K mode the cross term -> out[2 i + 1].
int launch_row_stats(Ctx& c, const float4* partials, int64_t Cn, float* out, int slot,
                     bool cross) {
  LaunchScope ls("row_reduce", c.st, 0, static_cast<double>(Cn) * c.pl.tiles_v * 16);
  row_reduce_kernel<<<static_cast<unsigned>(cdiv(Cn, 8)), 256, 0, c.st>>>(
      partials, c.pl.tiles_v, static_cast<int>(Cn), nullptr, nullptr, out + slot, nullptr, 2,
      cross ? out + 1 : nullptr);
  return KL_LAUNCHED();
}

// One CTA per logit row.  Top-K: 512 threads (4 CTAs per SM) beat 256 (8 per SM)
// by 3% on the bench chunk -- 4096 rows make 6.9 waves instead of 3.5, a
// smaller tail.  The full-vocabulary kernel streams two rows per CTA and was 1%
// slower at 512, so it keeps 256.
constexpr int kDlogitsThreads = 512;
constexpr int kDlogitsFullThreads = 256;

template <typename Elem>
int launch_dlogits_topk(Ctx& c, Elem* S, int64_t c0, int64_t Cn, const float* lse,
                        const float* g_dev, float g_host, const float4* part) {
  const kl_problem* p = c.p;
  static std::atomic<bool> attr[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev].load()) {
    cudaFuncSetAttribute(dlogits_topk_kernel<Elem>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kMaxK * 4);
    attr[dev].store(true);
  }
  LaunchScope ls("dlogits_topk", c.st, 0, 2.0 * Cn * p->V * sizeof(Elem));
  dlogits_topk_kernel<Elem><<<static_cast<unsigned>(Cn), kDlogitsThreads, p->K * 4, c.st>>>(
      S, c.pl.Vp, static_cast<int>(p->V), lse + c0, p->mask ? p->mask + c0 : nullptr,
      reinterpret_cast<const float2*>(c.ws + c.pl.off_rinfo),
      reinterpret_cast<const int*>(c.ws + c.pl.off_sidx),
      reinterpret_cast<const float*>(c.ws + c.pl.off_sq), p->K, c.sc, g_dev, g_host, c.invT,
      p->T_row ? p->T_row + c0 : nullptr, part, c.pl.tiles_v);
  return KL_LAUNCHED();
}

// dS in place over the student buffer, teacher-hidden mode (one CTA per row).
template <typename Elem>
int launch_dlogits_full(Ctx& c, Elem* S, const float* Tt, int64_t c0, int64_t Cn,
                        const float* lse_s, const float* lse_t, const float* ubar,
                        const float* g_dev, float g_host) {
  const kl_problem* p = c.p;
  LaunchScope ls("dlogits_full", c.st, 0, (2.0 * sizeof(Elem) + 4.0) * Cn * p->V);
  dlogits_full_kernel<Elem><<<static_cast<unsigned>(Cn), kDlogitsFullThreads, 0, c.st>>>(
      S, Tt, c.pl.Vp, static_cast<int>(p->V), lse_s + c0, lse_t + c0, ubar,
      p->mask ? p->mask + c0 : nullptr, c.sc, g_dev, g_host, c.invT,
      p->T_row ? p->T_row + c0 : nullptr, p->reverse_weight,
      reinterpret_cast<const float4*>(c.ws + c.pl.off_ps),
      reinterpret_cast<const float4*>(c.ws + c.pl.off_pt), c.pl.tiles_v);
  return KL_LAUNCHED();
}

// dS from the stored exponentials of chunk rows [c0, c0 + Cn) (top-K, bf16):
// the cached columns' corrections folded into the buffer S, then the
// transposed per-(tile, row) scales.  lse: the whole problem's rows.  Returns
// the scales for gemm_grads.
int launch_xf_prep(Ctx& c, __nv_bfloat16* S, int64_t c0, int64_t Cn, const float* lse,
                   const float* g_dev, float g_host, const float** xf_sc) {
  const kl_problem* p = c.p;
  const float4* part = reinterpret_cast<const float4*>(c.ws + c.pl.off_ps);
  const float2* rinfo = reinterpret_cast<const float2*>(c.ws + c.pl.off_rinfo);
  const uint8_t* mask = p->mask ? p->mask + c0 : nullptr;
  const float* T_row = p->T_row ? p->T_row + c0 : nullptr;
  float* sc_out = reinterpret_cast<float*>(c.ws + c.pl.off_xsc);
  {
    LaunchScope ls("xf_patch", c.st, 0, static_cast<double>(Cn) * p->K * 16);
    xf_patch_kernel<<<static_cast<unsigned>(cdiv(Cn, 8)), 256, 0, c.st>>>(
        S, c.pl.Vp, part, c.pl.tiles_v, static_cast<int>(Cn), static_cast<int>(p->V), lse + c0,
        mask, rinfo, reinterpret_cast<const int*>(c.ws + c.pl.off_sidx),
        reinterpret_cast<const float*>(c.ws + c.pl.off_sq), p->K, c.sc, g_dev, g_host, c.invT,
        T_row);
    KL_TRY(KL_LAUNCHED());
  }
  LaunchScope ls("xf_scales", c.st, 0, static_cast<double>(Cn) * c.pl.tiles_v * 20);
  xf_scales_kernel<<<static_cast<unsigned>(cdiv(Cn, 32)), 256, 0, c.st>>>(
      part, c.pl.tiles_v, static_cast<int>(Cn), lse + c0, mask, rinfo, c.sc, g_dev, g_host,
      c.invT, T_row, sc_out, c.pl.Cx);
  *xf_sc = sc_out;
  return KL_LAUNCHED();
}

// Teacher-hidden row sums of chunk rows [c0, c0 + Cn) (hidden_sums_kernel).
// lse_*_in: given log-sum-exps (whole arrays, or nullptr to merge them from the
// tile statistics into lse_*_out); the other outputs as the kernel's, each
// optional; sums_out / sums_all are per chunk ([rows] / [P][rows] pairs).
int launch_hidden_sums(Ctx& c, int64_t c0, int64_t Cn, const float* lse_s_in,
                       const float* lse_t_in, float* lse_s_out, float* lse_t_out, int add_lse,
                       float* row_loss, float* sums_out, float* ubar_out,
                       const float* sums_all = nullptr, int P = 1) {
  const kl_problem* p = c.p;
  LaunchScope ls("hidden_sums", c.st, 0, static_cast<double>(Cn) * c.pl.tiles_v * 32);
  hidden_sums_kernel<<<static_cast<unsigned>(cdiv(Cn, 8)), 256, 0, c.st>>>(
      reinterpret_cast<const float4*>(c.ws + c.pl.off_ps),
      reinterpret_cast<const float4*>(c.ws + c.pl.off_pt), c.pl.tiles_v, static_cast<int>(Cn),
      lse_s_in ? lse_s_in + c0 : nullptr, lse_t_in ? lse_t_in + c0 : nullptr,
      lse_s_out ? lse_s_out + c0 : nullptr, lse_t_out ? lse_t_out + c0 : nullptr,
      p->mask ? p->mask + c0 : nullptr, p->reverse_weight, add_lse,
      row_loss ? row_loss + c0 : nullptr, sums_out, ubar_out, sums_all, P);
  return KL_LAUNCHED();
}

// Teacher-hidden logits of one chunk: the teacher pass (fp32 t~ - tile max into
// the teacher buffer, statistics), then the student pass (statistics and the
// tile sums A, U formed against the teacher tile; s~ - tile max stored into
// the student buffer when store_student).
template <typename Elem>
int hidden_logits(Ctx& c, int64_t c0, int64_t Cn, bool store_student) {
  const kl_problem* p = c.p;
  float* Tt = reinterpret_cast<float*>(c.ws + c.pl.off_tbuf);
  float4* ps = reinterpret_cast<float4*>(c.ws + c.pl.off_ps);
  float4* pt = reinterpret_cast<float4*>(c.ws + c.pl.off_pt);
  KL_TRY(gemm_logits<Elem>(c, p->Ht, p->d_t, head_Wt(c), c0, Cn, Tt, true, pt,
                           nullptr, nullptr, 0, "gemm_teacher_logits"));
  return gemm_logits<Elem>(c, p->H, p->d, head_W(c), c0, Cn,
                           store_student ? c.ws + c.pl.off_sbuf : nullptr, sizeof(Elem) == 4, ps,
                           nullptr, nullptr, 0, "gemm_logits_stats", Tt, pt);
}

int launch_finalize(Ctx& c, const float* row_loss, float* loss) {
  LaunchScope ls("finalize_loss", c.st, 0, static_cast<double>(c.p->N) * 4);
  finalize_loss_kernel<<<1, 1024, 0, c.st>>>(row_loss, c.p->N, c.sc, loss);
  return KL_LAUNCHED();
}

int launch_fill(Ctx& c, float* p, int64_t n, float v) {
  if (n <= 0) return KL_OK;
  LaunchScope ls("fill", c.st, 0, static_cast<double>(n) * 4);
  fill_f32_kernel<<<static_cast<unsigned>(c.sms * 4), 256, 0, c.st>>>(p, n, v);
  return KL_LAUNCHED();
}

int begin(const kl_problem* p, int entry, void* ws, size_t ws_bytes, void* stream, Ctx& c,
          bool vocab_shard = false) {
  KL_TRY(validate(p));
  if (!vocab_shard && !whole_head(p)) return KL_ERR_ARG;
  DevInfo di;
  KL_TRY(current_device_info(&di));
  c.p = p;
  c.pl = make_plan(p, entry);
  if (ws == nullptr) return KL_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return KL_ERR_ALIGN;
  if (ws_bytes < c.pl.total) return KL_ERR_WORKSPACE;
  c.ws = static_cast<uint8_t*>(ws);
  c.sc = reinterpret_cast<Scalars*>(ws);
  c.st = static_cast<cudaStream_t>(stream);
  c.sms = di.sms;
  c.invT = 1.0f / p->T;
  return KL_OK;
}

// ------------------------------------------------------------------ entry bodies
template <typename Elem>
int run_fwd(Ctx& c, float* loss, float* lse_s, float* lse_t, float* row_loss) {
  const kl_problem* p = c.p;
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(c.ws + c.pl.off_rl);
  KL_TRY(launch_count_valid(c));
  KL_TRY(prepare_heads(c));
  float4* ps = reinterpret_cast<float4*>(c.ws + c.pl.off_ps);
  for (int64_t c0 = 0; c0 < p->N; c0 += c.pl.C) {
    const int64_t Cn = (p->N - c0) < c.pl.C ? (p->N - c0) : c.pl.C;
    // keep_last_chunk: the last chunk's logits stay in the student buffer
    const bool keep = p->keep_last_chunk && c0 + Cn == p->N;
    if (!c.pl.hidden) {
      KL_TRY(launch_prep(c, c0, Cn));
      KL_TRY(gemm_logits<Elem>(c, p->H, p->d, head_W(c), c0, Cn,
                               keep ? c.ws + c.pl.off_sbuf : nullptr, sizeof(Elem) == 4, ps,
                               reinterpret_cast<const int*>(c.ws + c.pl.off_sidx),
                               reinterpret_cast<const float*>(c.ws + c.pl.off_sq), p->K,
                               "gemm_logits_stats"));
      KL_TRY(launch_row_reduce(c, ps, c0, Cn, true, lse_s, rl));
    } else {
      KL_TRY(hidden_logits<Elem>(c, c0, Cn, keep));
      KL_TRY(launch_hidden_sums(c, c0, Cn, nullptr, nullptr, lse_s, lse_t, 1, rl, nullptr,
                                nullptr));
    }
  }
  return launch_finalize(c, rl, loss);
}

template <typename Elem>
int run_bwd(Ctx& c, const float* lse_s, const float* lse_t, const float* g_dev, float g_host,
            void* dH, float* dW, int accumulate) {
  const kl_problem* p = c.p;
  KL_TRY(launch_count_valid(c));  // also resets the status word
  if (p->N == 0) return accumulate ? KL_OK : launch_fill(c, dW, p->V * p->d, 0.f);
  Elem* S = reinterpret_cast<Elem*>(c.ws + c.pl.off_sbuf);
  KL_TRY(prepare_heads(c));
  if (sizeof(Elem) == 4)
    KL_TRY(launch_transpose(c, static_cast<const float*>(p->W), p->d,
                            reinterpret_cast<float*>(c.ws + c.pl.off_wT), c.pl.Vp, p->V, p->d));
  const int64_t nch = cdiv(p->N, c.pl.C);
  // keep_last_chunk: the last chunk first, from the logits kl_fwd left behind
  for (int64_t i = 0; i < nch; ++i) {
    const int64_t k = p->keep_last_chunk ? (i == 0 ? nch - 1 : i - 1) : i;
    const bool kept = p->keep_last_chunk && i == 0;
    const int64_t c0 = k * c.pl.C;
    const int64_t Cn = (p->N - c0) < c.pl.C ? (p->N - c0) : c.pl.C;
    if (!c.pl.hidden) {
      if (kept) {  // s~ - tile max, the tile statistics and the prepared cache are in ws
        KL_TRY(launch_dlogits_topk<Elem>(c, S, c0, Cn, lse_s, g_dev, g_host,
                                         reinterpret_cast<const float4*>(c.ws + c.pl.off_ps)));
      } else {
        KL_TRY(launch_prep(c, c0, Cn));
        KL_TRY(gemm_dlogits<Elem>(c, S, c0, Cn, lse_s, g_dev, g_host));
      }
    } else {
      // both logits recomputed (or kept); u_bar from the given lse's
      float* ubar = reinterpret_cast<float*>(c.ws + c.pl.off_ubar);
      if (!kept) KL_TRY(hidden_logits<Elem>(c, c0, Cn, true));
      KL_TRY(launch_hidden_sums(c, c0, Cn, lse_s, lse_t, nullptr, nullptr, 1, nullptr, nullptr,
                                ubar));
      KL_TRY(launch_dlogits_full<Elem>(c, S, reinterpret_cast<const float*>(c.ws + c.pl.off_tbuf),
                                       c0, Cn, lse_s, lse_t, ubar, g_dev, g_host));
    }
    KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, (accumulate || i > 0) ? 1 : 0));
  }
  return KL_OK;
}

template <typename Elem>
int run_fwd_bwd(Ctx& c, float g, float* loss, float* row_loss, void* dH, float* dW,
                int accumulate) {
  const kl_problem* p = c.p;
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(c.ws + c.pl.off_rl);
  float* lse_s = reinterpret_cast<float*>(c.ws + c.pl.off_lse_s);
  float* lse_t = c.pl.hidden ? reinterpret_cast<float*>(c.ws + c.pl.off_lse_t) : nullptr;
  Elem* S = reinterpret_cast<Elem*>(c.ws + c.pl.off_sbuf);
  float4* ps = reinterpret_cast<float4*>(c.ws + c.pl.off_ps);
  KL_TRY(launch_count_valid(c));
  if (p->N == 0) {
    if (!accumulate) KL_TRY(launch_fill(c, dW, p->V * p->d, 0.f));
    return launch_finalize(c, rl, loss);
  }
  KL_TRY(prepare_heads(c));
  if (sizeof(Elem) == 4)
    KL_TRY(launch_transpose(c, static_cast<const float*>(p->W), p->d,
                            reinterpret_cast<float*>(c.ws + c.pl.off_wT), c.pl.Vp, p->V, p->d));
  for (int64_t c0 = 0; c0 < p->N; c0 += c.pl.C) {
    const int64_t Cn = (p->N - c0) < c.pl.C ? (p->N - c0) : c.pl.C;
    const int beta = (accumulate || c0 > 0) ? 1 : 0;
    if (!c.pl.hidden) {
      KL_TRY(launch_prep(c, c0, Cn));
      KL_TRY(gemm_logits<Elem>(c, p->H, p->d, head_W(c), c0, Cn, S, sizeof(Elem) == 4, ps,
                               reinterpret_cast<const int*>(c.ws + c.pl.off_sidx),
                               reinterpret_cast<const float*>(c.ws + c.pl.off_sq), p->K,
                               "gemm_logits_stats", nullptr, nullptr, c.pl.xf));
      KL_TRY(launch_row_reduce(c, ps, c0, Cn, true, lse_s, rl));
      if (c.pl.xf) {  // fuse_dlogits: dS formed inside the dH contraction
        const float* xsc = nullptr;
        KL_TRY(launch_xf_prep(c, reinterpret_cast<__nv_bfloat16*>(S), c0, Cn, lse_s, nullptr, g,
                              &xsc));
        KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, beta, false, xsc));
        continue;
      }
      KL_TRY(launch_dlogits_topk<Elem>(c, S, c0, Cn, lse_s, nullptr, g, ps));
    } else {
      float* ubar = reinterpret_cast<float*>(c.ws + c.pl.off_ubar);
      KL_TRY(hidden_logits<Elem>(c, c0, Cn, true));
      KL_TRY(launch_hidden_sums(c, c0, Cn, nullptr, nullptr, lse_s, lse_t, 1, rl, nullptr, ubar));
      KL_TRY(launch_dlogits_full<Elem>(c, S, reinterpret_cast<const float*>(c.ws + c.pl.off_tbuf),
                                       c0, Cn, lse_s, lse_t, ubar, nullptr, g));
    }
    KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, beta));
  }
  return launch_finalize(c, rl, loss);
}

// ------------------------------------------------------------------ vocabulary-parallel chunks
// Rows [c0, c0 + Cn) of chunk k.
void chunk_rows(const Ctx& c, int64_t k, int64_t* c0, int64_t* Cn) {
  *c0 = k * c.pl.C;
  const int64_t left = c.p->N - *c0;
  *Cn = left < c.pl.C ? left : c.pl.C;
}

int64_t num_chunks(const kl_problem* p, int64_t C) { return p->N > 0 ? cdiv(p->N, C) : 0; }

template <typename Elem>
int run_vp_fwd_chunk(Ctx& c, int64_t k, float* stats) {
  const kl_problem* p = c.p;
  int64_t c0, Cn;
  chunk_rows(c, k, &c0, &Cn);
  if (k == 0) {  // start of a pass
    KL_TRY(launch_count_valid(c));
    KL_TRY(prepare_heads(c));
    if (sizeof(Elem) == 4)
      KL_TRY(launch_transpose(c, static_cast<const float*>(p->W), p->d,
                              reinterpret_cast<float*>(c.ws + c.pl.off_wT), c.pl.Vp, p->V, p->d));
  }
  Elem* S = reinterpret_cast<Elem*>(c.ws + c.pl.off_sbuf);
  float4* ps = reinterpret_cast<float4*>(c.ws + c.pl.off_ps);
  if (!c.pl.hidden) {
    KL_TRY(launch_prep(c, c0, Cn));
    KL_TRY(gemm_logits<Elem>(c, p->H, p->d, head_W(c), c0, Cn, S, sizeof(Elem) == 4, ps,
                             reinterpret_cast<const int*>(c.ws + c.pl.off_sidx),
                             reinterpret_cast<const float*>(c.ws + c.pl.off_sq), p->K,
                             "gemm_logits_stats", nullptr, nullptr, c.pl.xf));
    return launch_row_stats(c, ps, Cn, stats, 0, true);
  }
  float4* pt = reinterpret_cast<float4*>(c.ws + c.pl.off_pt);
  KL_TRY(hidden_logits<Elem>(c, c0, Cn, true));
  KL_TRY(launch_row_stats(c, ps, Cn, stats, 0, false));
  return launch_row_stats(c, pt, Cn, stats, 1, false);
}

// Merge the P shards' row statistics of chunk k: whole-vocabulary lse_s (and
// lse_t) into the workspace (and lse_user), and the top-K row-loss share.
int launch_vp_merge(Ctx& c, int64_t c0, int64_t Cn, const float* stats_all, int P, int rank,
                    float* lse_user, float* rl) {
  const kl_problem* p = c.p;
  float* lse_s = reinterpret_cast<float*>(c.ws + c.pl.off_lse_s);
  float* lse_t = c.pl.hidden ? reinterpret_cast<float*>(c.ws + c.pl.off_lse_t) : nullptr;
  LaunchScope ls("vp_merge", c.st, 0, static_cast<double>(Cn) * (8.0 * P + 12));
  vp_merge_kernel<<<static_cast<unsigned>(cdiv(Cn, 128)), 128, 0, c.st>>>(
      stats_all, P, static_cast<int>(Cn), c.pl.hidden ? 1 : 0, rank,
      p->mask ? p->mask + c0 : nullptr,
      c.pl.hidden ? nullptr : reinterpret_cast<const float2*>(c.ws + c.pl.off_rinfo),
      lse_s + c0, lse_t ? lse_t + c0 : nullptr, lse_user ? lse_user + c0 : nullptr, rl + c0);
  return KL_LAUNCHED();
}

// Teacher-hidden mode with a reverse-KL weight: this shard's sums (A, U) of
// chunk k over its columns, from the tile statistics and the whole-vocabulary
// lse's, written to sums_out [rows][2].
template <typename Elem>
int run_vp_mid_chunk(Ctx& c, int64_t k, const float* stats_all, int P, int rank,
                     float* sums_out) {
  int64_t c0, Cn;
  chunk_rows(c, k, &c0, &Cn);
  float* rl = reinterpret_cast<float*>(c.ws + c.pl.off_rl);
  KL_TRY(launch_vp_merge(c, c0, Cn, stats_all, P, rank, nullptr, rl));
  const float* lse_s = reinterpret_cast<const float*>(c.ws + c.pl.off_lse_s);
  const float* lse_t = reinterpret_cast<const float*>(c.ws + c.pl.off_lse_t);
  return launch_hidden_sums(c, c0, Cn, lse_s, lse_t, nullptr, nullptr, 0, nullptr, sums_out,
                            nullptr);
}

template <typename Elem>
int run_vp_bwd_chunk(Ctx& c, int64_t k, const float* stats_all, const float* sums_all, int P,
                     int rank, float g, float* loss, float* lse_user, float* row_loss, float* dH,
                     float* dW, int accumulate) {
  const kl_problem* p = c.p;
  int64_t c0, Cn;
  chunk_rows(c, k, &c0, &Cn);
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(c.ws + c.pl.off_rl);
  float* lse_s = reinterpret_cast<float*>(c.ws + c.pl.off_lse_s);
  float* lse_t = c.pl.hidden ? reinterpret_cast<float*>(c.ws + c.pl.off_lse_t) : nullptr;
  Elem* S = reinterpret_cast<Elem*>(c.ws + c.pl.off_sbuf);
  float4* ps = reinterpret_cast<float4*>(c.ws + c.pl.off_ps);
  const int beta = (accumulate || k > 0) ? 1 : 0;
  KL_TRY(launch_vp_merge(c, c0, Cn, stats_all, P, rank, lse_user, rl));
  if (!c.pl.hidden) {
    if (c.pl.xf) {  // fuse_dlogits: dS formed inside the dH contraction
      const float* xsc = nullptr;
      KL_TRY(launch_xf_prep(c, reinterpret_cast<__nv_bfloat16*>(S), c0, Cn, lse_s, nullptr, g,
                            &xsc));
      KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, beta, true, xsc));
    } else {
      KL_TRY(launch_dlogits_topk<Elem>(c, S, c0, Cn, lse_s, nullptr, g, ps));
      KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, beta, true));
    }
  } else {
    // this shard's A, U (its row-loss share) and u_bar, the sum of every shard's
    // U when the reverse KL needs it (its sums came through the second exchange)
    float* ubar = reinterpret_cast<float*>(c.ws + c.pl.off_ubar);
    const bool mixed = p->reverse_weight > 0.f;
    KL_TRY(launch_hidden_sums(c, c0, Cn, lse_s, lse_t, nullptr, nullptr, rank == 0 ? 1 : 0, rl,
                              nullptr, ubar, mixed ? sums_all : nullptr, P));
    KL_TRY(launch_dlogits_full<Elem>(c, S, reinterpret_cast<const float*>(c.ws + c.pl.off_tbuf),
                                     c0, Cn, lse_s, lse_t, ubar, nullptr, g));
    KL_TRY(gemm_grads<Elem>(c, S, c0, Cn, dH, dW, beta, true));
  }
  if (c0 + Cn == p->N) KL_TRY(launch_finalize(c, rl, loss));
  return KL_OK;
}

// Checks shared by the two vocabulary-parallel calls.
int vp_begin(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes, void* stream,
             Ctx& c) {
  KL_TRY(validate(p));
  if (p->keep_last_chunk) return KL_ERR_ARG;
  if (chunk < 0 || chunk >= num_chunks(p, make_plan(p, KL_ENTRY_FWD_BWD).C)) return KL_ERR_ARG;
  return begin(p, KL_ENTRY_FWD_BWD, ws, ws_bytes, stream, c, true);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

size_t kl_workspace_bytes(const kl_problem* p, int entry) {
  if (validate_shape(p) != KL_OK || entry < KL_ENTRY_FWD || entry > KL_ENTRY_FWD_BWD) return 0;
  return make_plan(p, entry).total;
}

int kl_fwd(const kl_problem* p, void* ws, size_t ws_bytes, float* loss, float* lse_s,
           float* lse_t, float* row_loss, void* stream) {
  if (p != nullptr && p->fuse_dlogits) return KL_ERR_ARG;
  Ctx c;
  KL_TRY(begin(p, KL_ENTRY_FWD, ws, ws_bytes, stream, c));
  if (loss == nullptr || (p->N > 0 && lse_s == nullptr) ||
      (p->N > 0 && p->teacher == KL_TEACHER_HIDDEN && lse_t == nullptr))
    return KL_ERR_NULL;
  return p->dtype == KL_DTYPE_BF16 ? run_fwd<__nv_bfloat16>(c, loss, lse_s, lse_t, row_loss)
                                   : run_fwd<float>(c, loss, lse_s, lse_t, row_loss);
}

int kl_bwd(const kl_problem* p, void* ws, size_t ws_bytes, const float* lse_s,
           const float* lse_t, const float* grad_loss, void* dH, float* dW, int accumulate_dW,
           void* stream) {
  if (p != nullptr && p->fuse_dlogits) return KL_ERR_ARG;
  Ctx c;
  KL_TRY(begin(p, KL_ENTRY_BWD, ws, ws_bytes, stream, c));
  if (dW == nullptr || grad_loss == nullptr ||
      (p->N > 0 && (dH == nullptr || lse_s == nullptr)) ||
      (p->N > 0 && p->teacher == KL_TEACHER_HIDDEN && lse_t == nullptr))
    return KL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(dH) | reinterpret_cast<uintptr_t>(dW)) & 15)
    return KL_ERR_ALIGN;
  return p->dtype == KL_DTYPE_BF16
             ? run_bwd<__nv_bfloat16>(c, lse_s, lse_t, grad_loss, 0.f, dH, dW, accumulate_dW)
             : run_bwd<float>(c, lse_s, lse_t, grad_loss, 0.f, dH, dW, accumulate_dW);
}

int kl_fwd_bwd(const kl_problem* p, void* ws, size_t ws_bytes, float grad_loss, float* loss,
               float* row_loss, void* dH, float* dW, int accumulate_dW, void* stream) {
  if (p != nullptr && p->keep_last_chunk) return KL_ERR_ARG;
  Ctx c;
  KL_TRY(begin(p, KL_ENTRY_FWD_BWD, ws, ws_bytes, stream, c));
  if (loss == nullptr || dW == nullptr || (p->N > 0 && dH == nullptr)) return KL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(dH) | reinterpret_cast<uintptr_t>(dW)) & 15)
    return KL_ERR_ALIGN;
  return p->dtype == KL_DTYPE_BF16
             ? run_fwd_bwd<__nv_bfloat16>(c, grad_loss, loss, row_loss, dH, dW, accumulate_dW)
             : run_fwd_bwd<float>(c, grad_loss, loss, row_loss, dH, dW, accumulate_dW);
}

int64_t kl_vp_num_chunks(const kl_problem* p) {
  if (validate_shape(p) != KL_OK) return -1;
  return num_chunks(p, make_plan(p, KL_ENTRY_FWD_BWD).C);
}

int kl_vp_fwd_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    float* row_stats, void* stream) {
  Ctx c;
  KL_TRY(vp_begin(p, chunk, ws, ws_bytes, stream, c));
  if (row_stats == nullptr) return KL_ERR_NULL;
  return p->dtype == KL_DTYPE_BF16 ? run_vp_fwd_chunk<__nv_bfloat16>(c, chunk, row_stats)
                                   : run_vp_fwd_chunk<float>(c, chunk, row_stats);
}

int kl_vp_mid_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    const float* row_stats_all, int P, int rank, float* sums, void* stream) {
  if (P < 1 || rank < 0 || rank >= P) return KL_ERR_ARG;
  if (p != nullptr && p->teacher != KL_TEACHER_HIDDEN) return KL_ERR_ARG;
  Ctx c;
  KL_TRY(vp_begin(p, chunk, ws, ws_bytes, stream, c));
  if (row_stats_all == nullptr || sums == nullptr) return KL_ERR_NULL;
  return p->dtype == KL_DTYPE_BF16
             ? run_vp_mid_chunk<__nv_bfloat16>(c, chunk, row_stats_all, P, rank, sums)
             : run_vp_mid_chunk<float>(c, chunk, row_stats_all, P, rank, sums);
}

int kl_vp_bwd_chunk(const kl_problem* p, int64_t chunk, void* ws, size_t ws_bytes,
                    const float* row_stats_all, const float* sums_all, int P, int rank,
                    float grad_loss, float* loss, float* lse_s, float* row_loss, float* dH_part,
                    float* dW, int accumulate_dW, void* stream) {
  if (P < 1 || rank < 0 || rank >= P) return KL_ERR_ARG;
  Ctx c;
  KL_TRY(vp_begin(p, chunk, ws, ws_bytes, stream, c));
  if (row_stats_all == nullptr || loss == nullptr || dH_part == nullptr || dW == nullptr ||
      (p->reverse_weight > 0.f && sums_all == nullptr))
    return KL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(dH_part) | reinterpret_cast<uintptr_t>(dW)) & 15)
    return KL_ERR_ALIGN;
  return p->dtype == KL_DTYPE_BF16
             ? run_vp_bwd_chunk<__nv_bfloat16>(c, chunk, row_stats_all, sums_all, P, rank,
                                               grad_loss, loss, lse_s, row_loss, dH_part, dW,
                                               accumulate_dW)
             : run_vp_bwd_chunk<float>(c, chunk, row_stats_all, sums_all, P, rank, grad_loss,
                                       loss, lse_s, row_loss, dH_part, dW, accumulate_dW);
}

int kl_cast_f32(const float* src, void* dst, int64_t n, int dtype, void* stream) {
  if (n < 0 || n % 4 != 0) return KL_ERR_SHAPE;
  if (dtype != KL_DTYPE_BF16 && dtype != KL_DTYPE_F32) return KL_ERR_DTYPE;
  if (n == 0) return KL_OK;
  if (src == nullptr || dst == nullptr) return KL_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15)
    return KL_ERR_ALIGN;
  DevInfo di;
  KL_TRY(current_device_info(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LaunchScope ls("cast_f32", st, 0, n * (dtype == KL_DTYPE_BF16 ? 6.0 : 8.0));
  const unsigned grid = static_cast<unsigned>(di.sms * 4);
  if (dtype == KL_DTYPE_BF16)
    cast_f32_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(src, static_cast<__nv_bfloat16*>(dst), n);
  else
    cast_f32_kernel<float><<<grid, 256, 0, st>>>(src, static_cast<float*>(dst), n);
  return KL_LAUNCHED();
}

int kl_status(void* ws, void* stream) {
  if (ws == nullptr) return KL_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return KL_ERR_CUDA;
  int s = 0;
  if (cudaMemcpy(&s, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KL_ERR_CUDA;
  return s;
}

const char* kl_status_string(int code) {
  switch (code) {
    case KL_OK: return "ok";
    case KL_ERR_NULL: return "a required pointer is NULL";
    case KL_ERR_SHAPE: return "a size is out of range";
    case KL_ERR_DTYPE: return "unknown dtype or teacher mode";
    case KL_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case KL_ERR_WORKSPACE: return "workspace smaller than kl_workspace_bytes()";
    case KL_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case KL_ERR_INDEX: return "top-K cache index out of range or duplicated";
    case KL_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case KL_ERR_UNSUPPORTED: return "the current device is not sm_100 (B200-class)";
    case KL_ERR_ARG: return "bad argument (temperature, chunk size or normaliser)";
    case KL_ERR_TOO_LARGE:
      return "problem needs more scratch than kl_fwd_noalloc's fixed array holds";
    default: return "unknown status";
  }
}

uint64_t kl_launch_count(void) { return g_launches.load(); }

int kl_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& k : g_prof)
    for (auto& e : k.ev) {
      g_ev_pool.push_back(e.first);
      g_ev_pool.push_back(e.second);
    }
  g_prof.clear();
  g_prof_on = true;
  return KL_OK;
}

int kl_profile_end(kl_profile_entry* out, int max_entries) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  int n = 0;
  for (auto& k : g_prof) {
    double ms = 0;
    for (auto& e : k.ev) {
      if (cudaEventSynchronize(e.second) != cudaSuccess) return -KL_ERR_CUDA;
      float t = 0;
      if (cudaEventElapsedTime(&t, e.first, e.second) != cudaSuccess) return -KL_ERR_CUDA;
      ms += t;
    }
    if (out != nullptr && n < max_entries) {
      kl_profile_entry& o = out[n];
      memset(&o, 0, sizeof(o));
      strncpy(o.name, k.name.c_str(), sizeof(o.name) - 1);
      o.launches = k.launches;
      o.total_ms = ms;
      o.flops = k.flops;
      o.bytes = k.bytes;
    }
    ++n;
  }
  return n;
}

}  // extern "C"

// ====================================================================== no-allocation forward
// Scratch for kl_fwd_noalloc: one fixed array in static device memory, so the
// call needs neither cudaMalloc nor a caller workspace.  Host code only names
// it through the address looked up below (the host-side symbol is a stand-in,
// not a device address).
static __device__ __align__(256) uint8_t g_noalloc_scratch[KL_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array for the current device and context.  It
// is looked up on every call (a cheap runtime query) rather than cached, so a
// context that was destroyed and created again never gets a stale address.
int noalloc_scratch(uint8_t** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
    return KL_ERR_CUDA;
  *out = static_cast<uint8_t*>(ptr);
  return KL_OK;
}
}  // namespace

extern "C" int kl_fwd_noalloc(const kl_problem* p, float* loss, float* lse_s, float* row_loss,
                              int* status, void* stream) {
  if (p != nullptr && (p->keep_last_chunk || p->fuse_dlogits)) return KL_ERR_ARG;
  KL_TRY(validate(p));
  if (!whole_head(p)) return KL_ERR_ARG;
  if (p->dtype != KL_DTYPE_BF16 || p->teacher != KL_TEACHER_TOPK) return KL_ERR_DTYPE;
  if (loss == nullptr || (p->N > 0 && (lse_s == nullptr || row_loss == nullptr)))
    return KL_ERR_NULL;
  DevInfo di;
  KL_TRY(current_device_info(&di));
  // Layout in the fixed array: scalars | tile statistics | sorted ids | q | (m, sum q log q).
  const int64_t tiles_v = cdiv(p->V, kBN);
  const size_t per_row = static_cast<size_t>(tiles_v) * sizeof(float4) +
                         static_cast<size_t>(p->K) * 8 + sizeof(float2);
  const size_t fixed = 256 + 4 * 256;  // header + alignment of the four regions
  if (per_row + fixed > KL_NOALLOC_SCRATCH_BYTES) return KL_ERR_TOO_LARGE;
  int64_t C = static_cast<int64_t>((KL_NOALLOC_SCRATCH_BYTES - fixed) / per_row);
  if (p->chunk_tokens > 0 && p->chunk_tokens < C) C = p->chunk_tokens;
  if (p->N < C) C = p->N > 0 ? p->N : 1;
  uint8_t* scratch = nullptr;
  KL_TRY(noalloc_scratch(&scratch));
  Ctx c;
  c.p = p;
  c.pl.eb = 2;
  c.pl.C = C;
  c.pl.Vp = cdiv(p->V, 8) * 8;
  c.pl.tiles_v = static_cast<int>(tiles_v);
  c.pl.hidden = false;
  size_t off = 256;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes);
    return o;
  };
  c.pl.off_ps = take(static_cast<size_t>(C) * tiles_v * sizeof(float4));
  c.pl.off_sidx = take(static_cast<size_t>(C) * p->K * 4);
  c.pl.off_sq = take(static_cast<size_t>(C) * p->K * 4);
  c.pl.off_rinfo = take(static_cast<size_t>(C) * sizeof(float2));
  c.pl.total = off;
  if (c.pl.total > KL_NOALLOC_SCRATCH_BYTES) return KL_ERR_TOO_LARGE;
  c.ws = scratch;
  c.sc = reinterpret_cast<Scalars*>(scratch);
  c.st = static_cast<cudaStream_t>(stream);
  c.sms = di.sms;
  c.invT = 1.0f / p->T;
  // run_fwd resets the status word first and overwrites every scratch region
  // before reading it, so the previous call's contents do not leak in.
  KL_TRY(run_fwd<__nv_bfloat16>(c, loss, lse_s, nullptr, row_loss));
  if (status != nullptr &&
      cudaMemcpyAsync(status, &c.sc->status, sizeof(int), cudaMemcpyDeviceToDevice, c.st) !=
          cudaSuccess)
    return KL_ERR_CUDA;
  return KL_OK;
}
