// kl_rowops.cuh -- the SIMT (HBM-bound) steps of the fused KL loss.
//
// Source: "Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and
// a Fused Chunked KL Loss", §3 "Offline distillation" (apart from the student's
// normaliser, every term of the top-K loss is a sum over the cached entries
// alone) and §3 "Offline implementations" (the chunked variant keeps one
// normaliser per token and adds its corrections at the cached positions only);
// KDFlow abstract for the teacher-hidden mode.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "kl_ptx.cuh"

namespace ckl {

constexpr int kStatusIndex = 7;  // KL_ERR_INDEX
constexpr int kStatusArg = 10;   // KL_ERR_ARG (a per-token temperature <= 0)

// 1 / T for a row: the row's own temperature when T_row is given.
__device__ __forceinline__ float row_invT(const float* T_row, int row, float invT) {
  return T_row != nullptr ? 1.f / T_row[row] : invT;
}
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kEmpty = 0x7fffffff;  // sorted-cache sentinel for an empty slot

// Scalars at the head of the workspace.
struct Scalars {
  int status;     // KL_OK or a device-detected error
  int n_valid;    // rows with mask = 1
  float norm;     // divisor of the loss mean (caller's normaliser or n_valid)
  float pad;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Round-to-nearest onto the tf32 grid (10 explicit mantissa bits).  The
// tensor cores read only those bits of an fp32 operand and drop the rest, which
// biases every product towards zero; operands of the fp32 path are rounded
// first so the error is unbiased.
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
// Value as it will be stored in an operand buffer of element type Elem.
template <typename Elem>
__device__ __forceinline__ float operand_round(float x) {
  return sizeof(Elem) == 4 ? round_tf32(x) : x;
}

template <typename Elem>
__device__ __forceinline__ float to_f(Elem x);
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <typename Elem>
__device__ __forceinline__ Elem from_f(float x);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ float from_f<float>(float x) {
  return x;
}

// Load / store 8 consecutive elements as one or two 16-byte vectors.
template <typename Elem>
__device__ __forceinline__ void load8(const Elem* src, float* f);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* src, float* f) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 b = reinterpret_cast<const float4*>(src)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
template <typename Elem>
__device__ __forceinline__ void store8(Elem* dst, const float* f);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* dst, const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float* f) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// Resets the status word and counts the rows that enter the mean.
__global__ void count_valid_kernel(const uint8_t* mask, int64_t N, float normalizer,
                                   const float* T_row, Scalars* sc) {
  __shared__ int part[32];
  __shared__ int badT;
  if (threadIdx.x == 0) badT = 0;
  __syncthreads();
  int c = 0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) {
    c += mask ? (mask[i] != 0) : 1;
    if (T_row != nullptr && !(T_row[i] > 0.f)) badT = 1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
    sc->status = badT ? kStatusArg : 0;
    sc->n_valid = tot;
    sc->norm = normalizer > 0.f ? normalizer : static_cast<float>(tot);
  }
}

// Per cached row (one warp per row): validate ids, sort the K entries by
// vocabulary id (empty slots last, as kEmpty), and turn teacher logits into
// probabilities on the support:
//   partial mass (lse_t != nullptr): q = exp(t / T - lse_t)
//   renormalised:                    q = softmax over valid entries of t / T
// rowinfo = (m = sum q, sum q log q), over all cached entries.
// Ids are vocabulary ids in [0, V_total).  The sorted ids are stored relative
// to this head's first row v_begin; entries outside [v_begin, v_begin + V_local)
// (another rank's vocabulary shard) become kBelow / kEmpty, so the sorted order
// holds and no column of this shard ever matches them.
constexpr int kBelow = static_cast<int>(0x80000000u);
__global__ void prep_topk_kernel(const int32_t* __restrict__ idx,
                                 const float* __restrict__ logit,
                                 const float* __restrict__ lse_t, float invT,
                                 const float* __restrict__ T_row, int V, int K, int rows,
                                 int* __restrict__ sidx, float* __restrict__ sq,
                                 float2* __restrict__ rowinfo, Scalars* sc, int v_begin,
                                 int V_local) {
  extern __shared__ int prep_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  int* key = prep_smem + warp * 3 * K;
  float* tv = reinterpret_cast<float*>(key + K);
  float* qv = tv + K;
  const int32_t* ri = idx + static_cast<int64_t>(row) * K;
  const float* rl = logit + static_cast<int64_t>(row) * K;
  bool bad = false;
  float tmax = -INFINITY;
  invT = row_invT(T_row, row, invT);
  for (int i = lane; i < K; i += 32) {
    int k = ri[i];
    if (k < -1 || k >= V) {
      bad = true;
      k = -1;
    }
    key[i] = k < 0 ? kEmpty : k;
    const float t = rl[i] * invT;
    tv[i] = t;
    if (k >= 0) tmax = fmaxf(tmax, t);
  }
  __syncwarp();
  float m = 0.f, negent = 0.f;
  if (lse_t != nullptr) {
    const float l = lse_t[row];
    for (int i = lane; i < K; i += 32) {
      const float q = key[i] != kEmpty ? expf(tv[i] - l) : 0.f;
      qv[i] = q;
      m += q;
      negent += q > 0.f ? q * logf(q) : 0.f;
    }
  } else {
    tmax = warp_max(tmax);
    float z = 0.f;
    for (int i = lane; i < K; i += 32) z += key[i] != kEmpty ? expf(tv[i] - tmax) : 0.f;
    z = warp_sum(z);
    const float lz = logf(z);
    for (int i = lane; i < K; i += 32) {
      const bool ok = key[i] != kEmpty && z > 0.f;
      const float q = ok ? expf(tv[i] - tmax) / z : 0.f;
      qv[i] = q;
      m += q;
      negent += (ok && q > 0.f) ? q * (tv[i] - tmax - lz) : 0.f;
    }
  }
  __syncwarp();
  m = warp_sum(m);
  negent = warp_sum(negent);
  int* so = sidx + static_cast<int64_t>(row) * K;
  float* qo = sq + static_cast<int64_t>(row) * K;
  for (int i = lane; i < K; i += 32) {
    const int ki = key[i];
    int rank = 0;
    for (int j = 0; j < K; ++j) {
      const int kj = key[j];
      rank += (kj < ki) || (kj == ki && j < i);
      bad |= (kj == ki && j != i && ki != kEmpty);
    }
    so[rank] = ki == kEmpty ? kEmpty
               : ki < v_begin ? kBelow
               : ki - v_begin >= V_local ? kEmpty
                                         : ki - v_begin;
    qo[rank] = qv[i];
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(&sc->status, 0, kStatusIndex);
  if (lane == 0) rowinfo[row] = make_float2(m, negent);
}

// Split-V merge (one warp per row): partials (max2, sumexp2, cross) of every
// 256-column tile -> lse = ln 2 * (M + log2 Z), written to lse_out[row * stride].
// In top-K mode also the row loss l = [sum q log q] - [sum q s~] + m * lse
// (0 on masked rows) when row_loss is given, and the cross term sum q s~ to
// cross_out[row * stride] when that is given (a vocabulary shard's statistics).
__global__ void row_reduce_kernel(const float4* __restrict__ partials, int tiles_n, int rows,
                                  const uint8_t* __restrict__ mask,
                                  const float2* __restrict__ rowinfo, float* __restrict__ lse_out,
                                  float* __restrict__ row_loss, int stride,
                                  float* __restrict__ cross_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const float4* pr = partials + static_cast<int64_t>(row) * tiles_n;
  float M = -INFINITY;
  for (int i = lane; i < tiles_n; i += 32) M = fmaxf(M, pr[i].x);
  M = warp_max(M);
  float Z = 0.f, cross = 0.f;
  for (int i = lane; i < tiles_n; i += 32) {
    const float4 v = pr[i];
    Z += v.y * ex2_approx(v.x - M);
    cross += v.z;
  }
  Z = warp_sum(Z);
  cross = warp_sum(cross);
  if (lane == 0) {
    const float lse = (M + log2f(Z)) * kLn2;
    lse_out[static_cast<int64_t>(row) * stride] = lse;
    if (cross_out != nullptr) cross_out[static_cast<int64_t>(row) * stride] = cross;
    if (rowinfo != nullptr && row_loss != nullptr) {
      const bool keep = mask == nullptr || mask[row] != 0;
      const float2 ri = rowinfo[row];
      row_loss[row] = keep ? (ri.y - cross + ri.x * lse) : 0.f;
    }
  }
}

__device__ __forceinline__ float grad_coef(const uint8_t* mask, int row, const Scalars* sc,
                                           const float* g_dev, float g_host, float invT,
                                           const float* T_row) {
  invT = row_invT(T_row, row, invT);
  const bool keep = mask == nullptr || mask[row] != 0;
  const float g = g_dev != nullptr ? *g_dev : g_host;
  const float norm = sc->norm;
  return (keep && norm > 0.f) ? g / norm * invT : 0.f;
}

// The logits epilogue stores s~ minus the row's maximum over the 256-column
// tile when it also records that tile's statistics (part != nullptr); this is
// the maximum to add back (base-2 units in part.x), or 0.
__device__ __forceinline__ float tile_max2(const float4* part, int row, int tiles_n, int col) {
  return part != nullptr ? part[static_cast<int64_t>(row) * tiles_n + (col >> 8)].x : 0.f;
}

// dS for the top-K loss, in place over the chunk's logit buffer (one CTA per
// row):  dS_j = c (m p_s,j - q_j [j in S]),  c = g / (n T),  p_s = exp(s~ - lse).
// The K cached positions are read before the dense pass and rewritten after it.
template <typename Elem>
__global__ void dlogits_topk_kernel(Elem* __restrict__ S, int64_t ld, int V,
                                    const float* __restrict__ lse, const uint8_t* __restrict__ mask,
                                    const float2* __restrict__ rowinfo,
                                    const int* __restrict__ sidx, const float* __restrict__ sq,
                                    int K, const Scalars* sc, const float* g_dev, float g_host,
                                    float invT, const float* __restrict__ T_row,
                                    const float4* __restrict__ part, int tiles_n) {
  extern __shared__ float sval[];
  const int row = blockIdx.x;
  Elem* srow = S + static_cast<int64_t>(row) * ld;
  const float coef = grad_coef(mask, row, sc, g_dev, g_host, invT, T_row);
  const int nvec = (V + 7) >> 3;
  if (coef == 0.f) {
    const float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) store8<Elem>(srow + v * 8, z);
    return;
  }
  const int* ri = sidx + static_cast<int64_t>(row) * K;
  const float* rq = sq + static_cast<int64_t>(row) * K;
  const float l2 = lse[row] * kLog2e;
  // sval[i]: base-2 exponent of p_s at cached entry i, read before the dense pass
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const int j = ri[i];  // in [0, V): a cached column of this head; else empty or elsewhere
    sval[i] = static_cast<unsigned>(j) < static_cast<unsigned>(V)
                  ? fmaf(to_f<Elem>(srow[j]), kLog2e, tile_max2(part, row, tiles_n, j) - l2)
                  : 0.f;
  }
  __syncthreads();
  const float m = rowinfo[row].x;
  const float cm = coef * m;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[8];
    load8<Elem>(srow + v * 8, f);
    const float off = tile_max2(part, row, tiles_n, v * 8) - l2;  // 8 | 256: one tile
#pragma unroll
    for (int i = 0; i < 8; ++i)
      f[i] = (v * 8 + i < V) ? operand_round<Elem>(cm * ex2_approx(fmaf(f[i], kLog2e, off)))
                             : 0.f;
    store8<Elem>(srow + v * 8, f);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const int j = ri[i];
    if (static_cast<unsigned>(j) < static_cast<unsigned>(V))
      srow[j] = from_f<Elem>(operand_round<Elem>(coef * (m * ex2_approx(sval[i]) - rq[i])));
  }
}

// dS from the stored exponentials (bf16 top-K, the opt-in fused-dS path).  The
// logits pass stores e_j = 2^(s~_j log2 e - M) with M the (row, 256-column tile) maximum
// (base 2), so the dense part of dS_j = c (m p_s,j - q_j [j in S]) is
// scale * e_j with
//   scale = c m 2^(max(M - lse log2 e, -64)),
// where c = g / (n T) (0 on masked rows).  The floor at 2^-64 keeps scale a
// normal float when a tile lies far below the row's maximum; the dense part it
// then adds, at most c m 2^-64 per entry, is far below any entry that matters.
// The correction -c q_j at a cached column is folded into the stored value
// itself (xf_patch_kernel), so that dS = scale * e everywhere and the dH
// contraction applies one factor per (row, tile) to its operand stages.
__device__ __forceinline__ float xf_scale(float cm, float M2, float l2) {
  return cm * ex2_approx(fmaxf(M2 - l2, -64.f));
}

// One warp per row, lanes over the K cached entries: e_j <- e_j - c q_j / scale
// at each cached column j of this head (bf16 stored exponentials in S, row
// stride ld), with scale as xf_scale for j's tile.  Reads the logits pass's
// tile maxima (part.x); masked rows and rows without cache mass keep e (their
// scale is 0).
__global__ void xf_patch_kernel(__nv_bfloat16* __restrict__ S, int64_t ld,
                                const float4* __restrict__ part, int tiles_n, int rows, int V,
                                const float* __restrict__ lse, const uint8_t* __restrict__ mask,
                                const float2* __restrict__ rowinfo,
                                const int* __restrict__ sidx, const float* __restrict__ sq,
                                int K, const Scalars* sc, const float* g_dev, float g_host,
                                float invT, const float* __restrict__ T_row) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const float c = grad_coef(mask, row, sc, g_dev, g_host, invT, T_row);
  const float cm = c * rowinfo[row].x;
  if (cm == 0.f) return;
  const float l2 = lse[row] * kLog2e;
  const int* ri = sidx + static_cast<int64_t>(row) * K;
  const float* rq = sq + static_cast<int64_t>(row) * K;
  __nv_bfloat16* srow = S + static_cast<int64_t>(row) * ld;
  for (int i = lane; i < K; i += 32) {
    const int j = ri[i];  // in [0, V): a cached column of this head; else empty or elsewhere
    if (static_cast<unsigned>(j) >= static_cast<unsigned>(V)) continue;
    const float scale =
        xf_scale(cm, part[static_cast<int64_t>(row) * tiles_n + (j >> 8)].x, l2);
    srow[j] = __float2bfloat16_rn(__bfloat162float(srow[j]) - c * rq[i] / scale);
  }
}

// Scales of dS (xf_scale) for the chunk's rows, transposed for the gradient
// contractions: sc_out[t * ld + row] for tile t.  A block covers 32 rows (lane
// = row, so the writes of each tile are contiguous) and its warps share the
// tiles.
__global__ void xf_scales_kernel(const float4* __restrict__ part, int tiles_n, int rows,
                                 const float* __restrict__ lse, const uint8_t* __restrict__ mask,
                                 const float2* __restrict__ rowinfo, const Scalars* sc,
                                 const float* g_dev, float g_host, float invT,
                                 const float* __restrict__ T_row, float* __restrict__ sc_out,
                                 int64_t ld) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 32 + lane;
  if (row >= rows) return;
  const float cm = grad_coef(mask, row, sc, g_dev, g_host, invT, T_row) * rowinfo[row].x;
  const float l2 = lse[row] * kLog2e;
  const float4* pr = part + static_cast<int64_t>(row) * tiles_n;
  for (int t = warp; t < tiles_n; t += blockDim.x >> 5)
    sc_out[static_cast<int64_t>(t) * ld + row] = xf_scale(cm, pr[t].x, l2);
}

// Teacher-hidden mode, one warp per row: from the tile statistics of the two
// logits passes -- student (max2, sumexp2, A_tile, U_tile) and teacher (max2,
// sumexp2, ., .), with A_tile = sum 2^(t - mt) (t~ - s~) and
// U_tile = sum 2^(s - ms) (s~ - t~) over the tile (fp32, formed in the student
// pass's epilogue) -- the row's
//   lse_s, lse_t (merged over the tiles, or given: lse_s_in / lse_t_in),
//   A = sum_j p_t,j (t~_j - s~_j) = sum_tiles 2^(mt - lse_t log2 e) A_tile,
//   U = sum_j p_s,j (s~_j - t~_j) = sum_tiles 2^(ms - lse_s log2 e) U_tile.
// Forward KL = A - lse_t + lse_s and reverse KL = U - lse_s + lse_t, so the row
// loss (1 - beta) KL(p_t || p_s) + beta KL(p_s || p_t) needs no other pass.
// Writes (each optional): lse_s_out / lse_t_out; row_loss (0 on masked rows;
// add_lse = 0 leaves the lse terms out: a vocabulary shard's share, whose A and
// U cover its own columns only); sums_out[row] = (A, U); ubar_out[row] = u_bar,
// the whole-vocabulary sum p_s (s~ - t~) that the reverse-KL gradient needs --
// U itself, or the sum of every shard's U from sums_all [P][rows][2] when given.
// Sums run in a fixed order.
__global__ void hidden_sums_kernel(const float4* __restrict__ part_s,
                                   const float4* __restrict__ part_t, int tiles_n, int rows,
                                   const float* __restrict__ lse_s_in,
                                   const float* __restrict__ lse_t_in, float* __restrict__ lse_s_out,
                                   float* __restrict__ lse_t_out, const uint8_t* __restrict__ mask,
                                   float beta, int add_lse, float* __restrict__ row_loss,
                                   float* __restrict__ sums_out, float* __restrict__ ubar_out,
                                   const float* __restrict__ sums_all, int P) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const float4* ps = part_s + static_cast<int64_t>(row) * tiles_n;
  const float4* pt = part_t + static_cast<int64_t>(row) * tiles_n;
  float lse_s, lse_t;  // natural units; the weights below use them in base 2
  if (lse_s_in != nullptr) {
    lse_s = lse_s_in[row];
    lse_t = lse_t_in[row];
  } else {
    float Ms = -INFINITY, Mt = -INFINITY;
    for (int i = lane; i < tiles_n; i += 32) {
      Ms = fmaxf(Ms, ps[i].x);
      Mt = fmaxf(Mt, pt[i].x);
    }
    Ms = warp_max(Ms);
    Mt = warp_max(Mt);
    float Zs = 0.f, Zt = 0.f;
    for (int i = lane; i < tiles_n; i += 32) {
      Zs += ps[i].y * ex2_approx(ps[i].x - Ms);
      Zt += pt[i].y * ex2_approx(pt[i].x - Mt);
    }
    // as row_reduce_kernel merges a row: the same bits as a caller-given lse
    lse_s = (Ms + log2f(warp_sum(Zs))) * kLn2;
    lse_t = (Mt + log2f(warp_sum(Zt))) * kLn2;
  }
  const float ls2 = lse_s * kLog2e, lt2 = lse_t * kLog2e;
  float A = 0.f, U = 0.f;
  for (int i = lane; i < tiles_n; i += 32) {
    const float4 s = ps[i];
    A += ex2_approx(pt[i].x - lt2) * s.z;
    U += ex2_approx(s.x - ls2) * s.w;
  }
  A = warp_sum(A);
  U = warp_sum(U);
  if (lane == 0) {
    if (lse_s_out != nullptr) lse_s_out[row] = lse_s;
    if (lse_t_out != nullptr) lse_t_out[row] = lse_t;
    if (sums_out != nullptr) {
      sums_out[2 * row] = A;
      sums_out[2 * row + 1] = U;
    }
    if (ubar_out != nullptr) {
      float ub = U;
      if (sums_all != nullptr) {
        const int64_t blk = static_cast<int64_t>(rows) * 2;
        ub = 0.f;
        for (int q = 0; q < P; ++q) ub += sums_all[q * blk + 2 * row + 1];
      }
      ubar_out[row] = ub;
    }
    if (row_loss != nullptr) {
      const bool keep = mask == nullptr || mask[row] != 0;
      const float dl = add_lse ? lse_s - lse_t : 0.f;
      row_loss[row] = keep ? (1.f - beta) * (A + dl) + beta * (U - dl) : 0.f;
    }
  }
}

// Full-vocabulary mode, dS in place over the student buffer (one CTA per row):
//   dS = c [(1 - beta)(p_s - p_t) + beta p_s (u - u_bar)],  u = s~ - t~,
// c = g / (n T) (0 on masked rows), with p_s from the stored s~ - ms (element
// type of H), p_t from the stored t~ - mt (fp32), the tile maxima (base 2)
// from the two passes' statistics, the row lse's and u_bar per row.  Columns
// from V to the row's padded end are written as 0.
template <typename Elem>
__global__ void dlogits_full_kernel(Elem* __restrict__ S, const float* __restrict__ Tt, int64_t ld,
                                    int V, const float* __restrict__ lse_s,
                                    const float* __restrict__ lse_t,
                                    const float* __restrict__ ubar,
                                    const uint8_t* __restrict__ mask, const Scalars* sc,
                                    const float* g_dev, float g_host, float invT,
                                    const float* __restrict__ T_row, float beta,
                                    const float4* __restrict__ part_s,
                                    const float4* __restrict__ part_t, int tiles_n) {
  const int row = blockIdx.x;
  Elem* srow = S + static_cast<int64_t>(row) * ld;
  const float* trow = Tt + static_cast<int64_t>(row) * ld;
  const float coef = grad_coef(mask, row, sc, g_dev, g_host, invT, T_row);
  const float ls2 = lse_s[row] * kLog2e, lt2 = lse_t[row] * kLog2e;
  const float cf = coef * (1.f - beta), cr = coef * beta;
  const float ub = beta > 0.f ? ubar[row] : 0.f;
  const int nvec = (V + 7) >> 3;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float fs[8], ft[8];
    load8<Elem>(srow + v * 8, fs);
    load8<float>(trow + v * 8, ft);
    // 8 | 256: the vector lies in one tile
    const float ms2 = part_s[static_cast<int64_t>(row) * tiles_n + (v >> 5)].x;
    const float mt2 = part_t[static_cast<int64_t>(row) * tiles_n + (v >> 5)].x;
    const float dshift = (ms2 - mt2) * kLn2;  // (s~ - t~) = (fs - ft) + dshift
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = v * 8 + i < V;
      const float pt = ex2_approx(fmaf(ft[i], kLog2e, mt2 - lt2));
      const float ps = ex2_approx(fmaf(fs[i], kLog2e, ms2 - ls2));
      const float g = cf * (ps - pt) + cr * ps * (((fs[i] - ft[i]) + dshift) - ub);
      fs[i] = in ? operand_round<Elem>(g) : 0.f;
    }
    store8<Elem>(srow + v * 8, fs);
  }
}

// Vocabulary-parallel merge (one thread per row).  stats holds, for each of P
// head shards (rank-major blocks of rows x 2 floats), the shard's row
// statistics: top-K mode (lse over the shard, cross term over the shard's
// cached entries); teacher-hidden mode (student lse, teacher lse over the
// shard).  A log-sum-exp over the union of shards is the log of the sum of the
// shards' exponentials; the cross term is a plain sum.  Shards merge in rank
// order, so every rank gets the same bits.  Writes the full-vocabulary lse_s
// (and lse_t) of each row, and in top-K mode the row loss
// [sum q log q] - cross + m * lse_s on rank 0 and 0 on the others (0 on masked
// rows), so that the ranks' row losses sum to the loss.
__global__ void vp_merge_kernel(const float* __restrict__ stats, int P, int rows, int hidden,
                                int rank, const uint8_t* __restrict__ mask,
                                const float2* __restrict__ rowinfo, float* __restrict__ lse_s,
                                float* __restrict__ lse_t, float* __restrict__ lse_copy,
                                float* __restrict__ row_loss) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const int64_t blk = static_cast<int64_t>(rows) * 2;
  float mx = -INFINITY, my = -INFINITY;
  for (int r = 0; r < P; ++r) {
    const float* st = stats + r * blk + static_cast<int64_t>(row) * 2;
    mx = fmaxf(mx, st[0]);
    my = fmaxf(my, st[1]);
  }
  float zx = 0.f, zy = 0.f, cross = 0.f;
  for (int r = 0; r < P; ++r) {
    const float* st = stats + r * blk + static_cast<int64_t>(row) * 2;
    zx += expf(st[0] - mx);
    if (hidden) zy += expf(st[1] - my);
    else cross += st[1];
  }
  const float ls = mx + logf(zx);
  lse_s[row] = ls;
  if (lse_copy != nullptr) lse_copy[row] = ls;
  if (hidden) {
    lse_t[row] = my + logf(zy);
  } else if (row_loss != nullptr) {
    const bool keep = mask == nullptr || mask[row] != 0;
    const float2 ri = rowinfo[row];
    row_loss[row] = (keep && rank == 0) ? (ri.y - cross + ri.x * ls) : 0.f;
  }
}

// dst = src converted to Elem, n values (n a multiple of 4).
template <typename Elem>
__global__ void cast_f32_kernel(const float* __restrict__ src, Elem* __restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < (n >> 2);
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[i];
    dst[4 * i] = from_f<Elem>(a.x);
    dst[4 * i + 1] = from_f<Elem>(a.y);
    dst[4 * i + 2] = from_f<Elem>(a.z);
    dst[4 * i + 3] = from_f<Elem>(a.w);
  }
}

// loss = sum_n row_loss[n] / norm, summed in fp64 in a fixed order.
__global__ void finalize_loss_kernel(const float* __restrict__ row_loss, int64_t N,
                                     const Scalars* sc, float* loss) {
  __shared__ double red[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) s += row_loss[i];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    a = warp_sum_d(a);
    if (threadIdx.x == 0) *loss = sc->norm > 0.f ? static_cast<float>(a / sc->norm) : 0.f;
  }
}

// dst[c][r] = tf32-rounded src[r][c] for a rows x cols fp32 block (32 x 32
// smem tiles).  tf32 operands are kept K-major: the 128-byte swizzle does not
// serve MN-major 32-bit operands, so the fp32 path transposes them instead.
__global__ void transpose_f32_kernel(const float* __restrict__ src, int64_t ld_src,
                                     float* __restrict__ dst, int64_t ld_dst, int rows,
                                     int cols) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < rows && c < cols) ? src[static_cast<int64_t>(r) * ld_src + c] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows)
      dst[static_cast<int64_t>(c) * ld_dst + r] = round_tf32(tile[threadIdx.x][i]);
  }
}

// dst = tf32-rounded src for `rows` rows of `cols` fp32 values (row strides
// ld_src, ld_dst).
__global__ void round_tf32_kernel(const float* __restrict__ src, int64_t ld_src,
                                  float* __restrict__ dst, int64_t ld_dst, int64_t rows,
                                  int64_t cols) {
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    dst[r * ld_dst + c] = round_tf32(src[r * ld_src + c]);
  }
}

// out = sum over parts s = 0..S-1 of part[s] (fixed order), converted to Elem;
// rows x cols values, part slices `slice` elements apart, row stride ld.
template <typename Elem>
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int S, int64_t slice,
                                     Elem* __restrict__ out, int64_t n) {
  const int64_t nv = n >> 2;  // n is a multiple of 8 (rows of d, d % 8 == 0)
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < S; ++s) {
      const float4 b = reinterpret_cast<const float4*>(part + s * slice)[i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    const float f[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) out[i * 4 + k] = from_f<Elem>(f[k]);
  }
}

__global__ void fill_f32_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

}  // namespace ckl
