// kl_gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for the three
// contractions of the fused KL loss, with the loss arithmetic fused into the
// epilogue and, optionally, into the dH contraction's operand path
// ("Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and a
// Fused Chunked KL Loss", §3 "Fused chunked KL": the output projection is
// integrated into the loss and each logit chunk is transient).
//
//   C[M, N] = A[M, K] . B[N, K]^T   (bf16 -> kind::f16, fp32 -> kind::tf32;
//                                     fp32 accumulation in TMEM)
//
//   EPI_STATS  logits tile S = H_c . W^T: per (row, 256-column tile) the
//              max and sum of 2^(s~ log2 e - max) and the cross term
//              sum_i q_i s~_{idx_i} of the cached top-K entries that fall in
//              the tile (gathered from the fp32 accumulator).  Optionally
//              stores s~ - max (store = 1; natural units; fp32 or the input
//              type) or the exponentials 2^(s~ log2 e - max) themselves
//              (store = 2), which the dH contraction then scales into dS as its
//              operand stages arrive (XF, the opt-in fused-dS path).  In
//              the teacher-hidden mode the student pass also reads the
//              teacher tile (stored fp32 by the teacher pass) and forms the
//              tile's sums sum p_t (t~ - s~) and sum p_s (s~ - t~) from fp32.
//   EPI_STORE  dH_c = dS . W    -> element type of H, clipped to the chunk.
//   EPI_ACCUM  dW  (+)= dS^T . H_c -> fp32, add-reduced into dW across chunks;
//              also the fp32 split-K parts of dH.
//   EPI_DLOGITS backward with the row lse already known (the split forward /
//              backward path): dS = c (m exp(s~ - lse) - q [j in S]) formed from
//              the fp32 accumulator and stored, with c = g / (n T) (0 on masked
//              rows) -- no logits are stored and no separate dlogits pass runs.
//
// Two tile shapes: PAIR = 0, one CTA computes a 128 x 256 tile with
// tcgen05.mma.cta_group::1; PAIR = 1, a cluster of two CTAs (one per SM)
// computes a 256 x 256 tile with tcgen05.mma.cta_group::2: each CTA loads its
// own 128 rows of A and its own 128-row half of B, only the leader CTA issues
// the MMAs, the leader's commits arrive on both CTAs' barriers, and each CTA's
// epilogue reads its own 128 accumulator rows from its own TMEM.  The pair
// halves the operand bytes each SM stages per MMA.
//
// Roles (192 threads, 320 with XF or EG = 2; one CTA per SM, grid-strided over
// output tiles):
//   warps 0-3  epilogue: thread t of warp w owns accumulator row 32 (w mod 4) + t
//              (TMEM lane), reads 32 fp32 columns per tcgen05.ld;
//   warp 4     TMA producer (one thread): STAGES-deep ring of A/B tiles;
//   warp 5     TMEM allocator + MMA issuer (one thread);
//   warps 6-9  (XF = 1 only, dH) operand transform: turn the A stage -- the
//              stored exponentials e = 2^(s~ log2 e - tile max) of a logit
//              chunk, already corrected at the cached entries -- into
//              dS = scale(row, tile) * e in shared memory before the MMAs read
//              it, and store the formed stage as the dS chunk that the dW
//              contraction then reads.  This is the dlogits step of the loss
//              without its own pass over HBM (measured slower than that pass
//              on B200 at d >= 2048, so it is opt-in).
//   warps 6-9  (EG = 2 only, the teacher-hidden student pass) a second group
//              of epilogue warps, taking every other unit.
// Two 256-column accumulators in TMEM (512 columns) let the epilogue of tile
// i overlap the main loop of tile i + 1; the WIDE variant (dH) instead fills
// the 512 columns with one 256 x 512 tile (see the template below).  Waiting
// threads are parked by the hardware between barrier polls rather than
// spinning.
//
// Every wait on an mbarrier is bounded (spin_limit clock cycles); when one
// runs out the CTA records KL_ERR_TIMEOUT in *status and raises the abort flag
// of both CTAs of its pair, every role leaves its loop, the MMAs already
// issued are drained, and after both CTAs of the pair have stopped, the copies
// already issued are drained (again with a bound) before TMEM is released and
// the CTAs exit.
#pragma once
#include <cuda_bf16.h>

#include "kl_ptx.cuh"

namespace ckl {

constexpr int kBM = 128;          // tile rows (TMEM lanes)
constexpr int kBN = 256;          // tile columns (TMEM columns per accumulator)
constexpr int kStages = 4;        // smem ring depth (1-CTA tiles)
constexpr int kStagesPair = 6;    // smem ring depth (2-CTA tiles: 32 KB stages)
constexpr int kRowBytes = 128;    // one 128-B swizzle span per tile row / slab row
constexpr int kATileBytes = kBM * kRowBytes;
constexpr int kBTileBytes = kBN * kRowBytes;
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kGemmThreads = 192;
constexpr int kGemmThreadsXf = 320;  // + four operand-transform warps
constexpr int kTmemCols = 2 * kBN;
constexpr int kRingBytes = kStages * kStageBytes;          // 192 KB operand ring
constexpr int kBarrierRegion = 1024;                        // barriers, TMEM slot, flags
constexpr int kStageOutBytes = 4096;                        // one 32 x 32 fp32 output box
constexpr int kStagingBytes = 4 * 2 * kStageOutBytes;       // 4 epilogue warps x 2 buffers
constexpr int kGemmSmemBytes = 1024 /*align*/ + kRingBytes + kBarrierRegion + kStagingBytes;
static_assert(kStagesPair * (kATileBytes + kBTileBytes / 2) <= kRingBytes,
              "pair ring must fit the same shared-memory budget");
static_assert(kGemmSmemBytes <= 232448, "shared memory per CTA");

constexpr int kStatusTimeout = 8;  // KL_ERR_TIMEOUT
// Bound of the waits that drain in-flight copies and MMAs after an abort.  It
// does not shrink with the caller's spin limit: those copies and MMAs always
// finish on their own, and the CTA must not leave before they do.
constexpr long long kDrainLimit = 1LL << 31;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2f = 0.6931471805599453f;

enum { EPI_STATS = 0, EPI_STORE = 1, EPI_ACCUM = 2, EPI_DLOGITS = 3 };
// EPI_STATS store modes
enum { STORE_NONE = 0, STORE_SHIFTED = 1, STORE_EXP = 2 };

struct GemmParams {
  int tiles_m, tiles_n, num_kb;  // tiles_m counts 256-row tiles when PAIR = 1
  int m_fastest;       // raster: consecutive tile ids walk M first (else N first)
  int store;           // STATS: STORE_NONE / STORE_SHIFTED / STORE_EXP
  int out_f32;         // STATS, STORE_SHIFTED: the output map holds fp32
  int rows_valid;      // output rows that exist (M extent)
  int cols_valid;      // output columns that exist (N extent)
  float scale;         // STATS / DLOGITS: 1 / T
  const float* T_row;  // STATS / DLOGITS: per-row temperature (chunk rows), or nullptr
  int beta;            // ACCUM: 0 overwrite, 1 accumulate
  float4* partials;    // STATS: [rows][tiles_n] (max2, sumexp2, cross | A, 0 | U)
  const int* sidx;     // STATS gather: [rows][ktop] ascending ids, INT_MAX = empty
  const float* sq;     // STATS gather: [rows][ktop] teacher probabilities
  int ktop;            // STATS gather: entries per row (0 = no gather)
  // STATS, student pass of the teacher-hidden mode: the teacher tile stored by
  // the teacher pass (t~ - tile max, fp32, row stride tld) and its statistics
  const float* tbuf;
  int64_t tld;
  const float4* tpart;
  // XF: scale of dS per (256-column tile, logit row), [tiles][xf_ld] fp32
  // (xf_ld a multiple of 64), so that dS = scale * e for the stored e
  const float* xf_sc;
  int64_t xf_ld;
  int xf_rows;         // logit rows (tokens) that exist
  int xf_store;        // XF: store each formed dS stage through the fourth map (the
                       // dS chunk for dW); each row by one output column tile
  // DLOGITS: per-row lse (natural units), (m, .) per row, mask, and the scalars
  // of c = g / (n T): the loss normaliser n, and g (device pointer or value)
  const float* lse;
  const float2* rowinfo;
  const uint8_t* mask;
  const float* norm;
  const float* g_dev;
  float g_host;
  int ksplit = 1;      // split of the K range into ksplit contiguous parts (>= 1)
  int split_rows = 0;  // ACCUM with ksplit > 1: output-map rows between the parts' outputs
  int* status;         // device status word
  long long spin_limit;
};

// Work unit u covers output tile (u mod tiles) and K-part (u div tiles); the
// host guarantees every part is non-empty.
struct UnitRange {
  int tile, ks, kb0, kb1;
};
__device__ __forceinline__ UnitRange unit_range(int u, const GemmParams& p) {
  const int tiles = p.tiles_m * p.tiles_n;
  const int kbs = (p.num_kb + p.ksplit - 1) / p.ksplit;
  UnitRange r;
  r.tile = u % tiles;
  r.ks = u / tiles;
  r.kb0 = r.ks * kbs;
  r.kb1 = min(p.num_kb, r.kb0 + kbs);
  return r;
}

struct Ctl {
  int* status;
  long long limit;
  volatile int* abort_flag;
  uint32_t peer_abort;  // shared::cluster address of the other CTA's flag (0: none)
};

// Bounded wait for the phase of the given parity; false when the CTA aborted.
// park: let the hardware park the waiting thread between polls.
constexpr uint32_t kParkNs = 100;
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Ctl& c,
                                         bool park = false) {
  auto poll = [&]() {
    return park ? mbar_try_wait_suspend(bar, parity, kParkNs) : mbar_try_wait(bar, parity);
  };
  if (poll()) return true;
  const long long t0 = clock64();
  while (!poll()) {
    if (*c.abort_flag) return false;
    if (clock64() - t0 > c.limit) {
      *c.abort_flag = 1;
      if (c.peer_abort != 0u) st_cluster_u32(c.peer_abort, 1u);  // stop the pair together
      atomicCAS(c.status, 0, kStatusTimeout);
      return false;
    }
  }
  return true;
}

template <typename Elem>
struct ElemTraits;
template <>
struct ElemTraits<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr uint32_t kFmt = 1;  // bf16
};
template <>
struct ElemTraits<float> {
  static constexpr int kBytes = 4;
  static constexpr uint32_t kFmt = 2;  // tf32
};

// Round-to-nearest onto the tf32 grid (for dS stored as an fp32 tf32 operand).
__device__ __forceinline__ float round_tf32_dev(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& tm, int& tn) {
  if (p.m_fastest) {
    tm = t % p.tiles_m;
    tn = t / p.tiles_m;
  } else {
    tn = t % p.tiles_n;
    tm = t / p.tiles_n;
  }
}

// Pack 8 consecutive fp32 values into one 16-byte vector of Elem.
template <typename Elem>
__device__ __forceinline__ void store_vec(Elem* dst, const float* v);
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16>(__nv_bfloat16* dst, const float* v) {
  __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
  uint4 u;
  u.x = *reinterpret_cast<uint32_t*>(&h0);
  u.y = *reinterpret_cast<uint32_t*>(&h1);
  u.z = *reinterpret_cast<uint32_t*>(&h2);
  u.w = *reinterpret_cast<uint32_t*>(&h3);
  *reinterpret_cast<uint4*>(dst) = u;
}
template <>
__device__ __forceinline__ void store_vec<float>(float* dst, const float* v) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// XF: one 128-byte row of a dS operand stage (64 bf16 values of one logit row
// within one 256-column tile), x -> x * scale in place with packed bf16x2
// multiplies (scale rounded to bf16: with the product's rounding, 2^-8
// relative error per entry).  The chunks are visited in the row's swizzled
// order (chunk j at position j ^ sw) so that the 32 rows a warp's lanes touch
// at once hit all 32 banks.
__device__ __forceinline__ void xf_row(uint8_t* rowp, int sw, __nv_bfloat162 scale2) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint4* cp = reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4));
    uint4 u = *cp;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __hmul2(h[i], scale2);
    *cp = u;
  }
}

// WIDE = 1 (2-CTA pairs, store / accumulate epilogues): each work unit is a
// 256 x 512 output tile computed as two N = 256 MMAs per K step that share the
// A stage, so a CTA pulls 25% fewer operand bytes from L2 per MMA.  Both halves
// fill all 512 TMEM columns, so there is a single accumulator: the next unit's
// MMAs wait for the epilogue (worth it where units are long, as in dH).
// XF = 1 (dH: 2-CTA pairs, bf16, K-major A, store / accumulate epilogues): the
// A operand is a stage of stored exponentials that the transform warps turn
// into dS.  Each CTA's copies then complete on its own barriers (the transform
// warps of both CTAs wait for them), the MMA issuer waits for the transforms
// of both CTAs on a third ring of barriers, and a stage is refilled only after
// the MMAs and the transform warps' dS stores (tmD) have read it.
// EG = 2 (bf16 statistics epilogues with a heavy per-element tail, the
// student pass of the teacher-hidden mode): a second group of four epilogue
// warps (6-9).  Group g takes every other unit of the CTA -- always the one
// whose accumulator is TMEM buffer g -- so each unit's epilogue may last two
// units' worth of MMAs.  The staging boxes are bf16 (2 KB).
template <typename Elem, int A_MN, int B_MN, int EPI, int PAIR, int WIDE = 0, int XF = 0,
          int EG = 1>
__global__ void __launch_bounds__((XF || EG == 2) ? kGemmThreadsXf : kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
  static_assert(!WIDE || (PAIR && (EPI == EPI_STORE || EPI == EPI_ACCUM)),
                "wide tiles: 2-CTA pairs with a store or accumulate epilogue");
  static_assert(!XF || (PAIR && sizeof(Elem) == 2 && A_MN == 0 &&
                        (EPI == EPI_STORE || EPI == EPI_ACCUM)),
                "operand transform: bf16 2-CTA pairs, K-major A, store or accumulate");
  static_assert(EG == 1 || (EG == 2 && EPI == EPI_STATS && PAIR && !WIDE && !XF &&
                            sizeof(Elem) == 2),
                "two epilogue groups: bf16 statistics epilogues on 2-CTA pairs");
  constexpr int kCtas = PAIR ? 2 : 1;
  constexpr int kHalves = WIDE ? 2 : 1;               // N = 256 MMAs per K step
  constexpr int kTileN = kBN * kHalves;               // output columns per unit
  constexpr int kAccBufs = WIDE ? 1 : 2;              // accumulators in TMEM
  // Waiting threads let the hardware park them between polls (a 100 ns hint):
  // the producer, MMA and epilogue threads stop spinning, which under the power
  // cap made logits 10% and dW 3% faster.  With the short hint the wake-up
  // latency no longer costs the single-accumulator wide tiles either.
  constexpr bool kPark = true;
  constexpr int kBRows = kBN / kCtas;                 // B rows per half staged by this CTA
  constexpr int kBBytes = kBRows * kRowBytes;
  constexpr int kSBytes = kATileBytes + kHalves * kBBytes;  // this CTA's stage bytes
  constexpr int kNS = PAIR ? (WIDE ? kRingBytes / kSBytes : kStagesPair) : kStages;  // ring
  constexpr int kEB = ElemTraits<Elem>::kBytes;
  constexpr int kBKe = kRowBytes / kEB;       // K elements per stage (64 / 32)
  constexpr int kUmmaK = 32 / kEB;            // K per MMA instruction (16 / 8)
  constexpr int kKSteps = kBKe / kUmmaK;      // 4
  constexpr int kMNe = kRowBytes / kEB;       // MN elements per MN-major slab
  constexpr int kSlabBytes = kBKe * kRowBytes;
  constexpr uint32_t kIdesc =
      idesc_dense(ElemTraits<Elem>::kFmt, kBM * kCtas, kBN, A_MN, B_MN);
  // copies of each CTA complete on its own barriers (else on the leader's)
  constexpr bool kLocalCopies = XF || !PAIR;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kRingBytes);
  uint8_t* staging = smem + kRingBytes + kBarrierRegion;  // 1024-B aligned
  uint64_t* empty_bar = full_bar + kNS;
  uint64_t* ready_bar = empty_bar + kNS;  // XF: stage transformed in both CTAs
  uint64_t* tfull_bar = ready_bar + kNS;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* issued_slot = tmem_slot + 2;  // stages whose copies this CTA's producer issued

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = p.tiles_m * p.tiles_n * p.ksplit;  // work units
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // CTA rank within the pair
  const bool leader = rank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], XF ? 1 + 4 : 1);  // MMA commit (+ each transform warp)
      mbar_init(&ready_bar[s], 4 * kCtas);        // one arrival per transform warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 4 * kCtas);  // one arrival per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *issued_slot = 0u;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 5) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
    tc_fence_before();
  }
  __syncthreads();
  if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort =
      PAIR ? mapa_shared(const_cast<int*>(abort_flag), rank ^ 1u) : 0u;
  const Ctl ctl{p.status, p.spin_limit, abort_flag, peer_abort};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0;
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += units) {
        const UnitRange ur = unit_range(t, p);
        int tm, tn;
        tile_coords(ur.tile, p, tm, tn);
        const int m0 = tm * kBM * kCtas + static_cast<int>(rank) * kBM;  // this CTA's A rows
        const int n0 = tn * kTileN + static_cast<int>(rank) * kBRows;     // this CTA's B rows
        for (int kb = ur.kb0; kb < ur.kb1; ++kb) {
          const uint32_t s = issued % kNS;
          const uint32_t ph = (issued / kNS) & 1u;
          if (!wait_bar(&empty_bar[s], ph ^ 1u, ctl, kPark)) {
            ok = false;
            break;
          }
          uint8_t* a_s = smem + s * kSBytes;
          uint8_t* b_s = a_s + kATileBytes;
          if (kLocalCopies) mbar_arrive_expect_tx(&full_bar[s], kSBytes);
          else if (leader) mbar_arrive_expect_tx(&full_bar[s], kSBytes * kCtas);
          const uint32_t fb = kLocalCopies ? 0u : mapa_shared(&full_bar[s], 0);
          const int k0 = kb * kBKe;
#pragma unroll
          for (int sl = 0; sl < (A_MN ? kBM / kMNe : 1); ++sl) {
            void* dst = a_s + sl * kSlabBytes;
            const int x = A_MN ? m0 + sl * kMNe : k0, y = A_MN ? k0 : m0;
            if (kLocalCopies) tma_load_2d(&tmA, &full_bar[s], dst, x, y);
            else tma_load_2d_pair(&tmA, fb, dst, x, y);
          }
#pragma unroll
          for (int h = 0; h < kHalves; ++h) {
            const int nh = n0 + h * kBN;  // this CTA's B rows of half h
#pragma unroll
            for (int sl = 0; sl < (B_MN ? kBRows / kMNe : 1); ++sl) {
              void* dst = b_s + h * kBBytes + sl * kSlabBytes;
              const int x = B_MN ? nh + sl * kMNe : k0, y = B_MN ? k0 : nh;
              if (kLocalCopies) tma_load_2d(&tmB, &full_bar[s], dst, x, y);
              else tma_load_2d_pair(&tmB, fb, dst, x, y);
            }
          }
          ++issued;
        }
      }
      *issued_slot = issued;
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      uint32_t consumed = 0, local = 0;
      bool ok = true;
      for (int t = unit; t < total_tiles && ok; t += units, ++local) {
        const uint32_t buf = local % kAccBufs;
        const uint32_t aph = (local / kAccBufs) & 1u;
        if (!wait_bar(&tempty_bar[buf], aph ^ 1u, ctl, kPark)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kBN;
        const UnitRange ur = unit_range(t, p);
        for (int kb = ur.kb0; kb < ur.kb1; ++kb) {
          const uint32_t s = consumed % kNS;
          const uint32_t ph = (consumed / kNS) & 1u;
          const bool got = XF ? wait_bar(&ready_bar[s], ph, ctl, kPark)
                              : wait_bar(&full_bar[s], ph, ctl, kPark);
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kSBytes);
          const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
          for (int j = 0; j < kKSteps; ++j) {
            const uint64_t ad = A_MN ? sdesc_sw128(a_addr + j * (kUmmaK / 8) * 1024,
                                                   kSlabBytes, 1024)
                                     : sdesc_sw128(a_addr + j * 32, 16, 1024);
            const uint32_t acc = (kb != ur.kb0 || j != 0) ? 1u : 0u;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
              const uint32_t bh = b_addr + h * kBBytes;
              const uint64_t bd = B_MN ? sdesc_sw128(bh + j * (kUmmaK / 8) * 1024,
                                                     kSlabBytes, 1024)
                                       : sdesc_sw128(bh + j * 32, 16, 1024);
              const uint32_t dh = d_tmem + h * kBN;
              if (PAIR) {
                if (kEB == 2) umma_f16_pair(dh, ad, bd, kIdesc, acc);
                else umma_tf32_pair(dh, ad, bd, kIdesc, acc);
              } else {
                if (kEB == 2) umma_f16(dh, ad, bd, kIdesc, acc);
                else umma_tf32(dh, ad, bd, kIdesc, acc);
              }
            }
          }
          // frees the smem stage (in both CTAs of a pair) when these MMAs finish
          if (PAIR) umma_commit_pair(&empty_bar[s], 0x3);
          else umma_commit(&empty_bar[s]);
          ++consumed;
        }
        if (!ok) break;
        // accumulator ready for the epilogue(s)
        if (PAIR) umma_commit_pair(&tfull_bar[buf], 0x3);
        else umma_commit(&tfull_bar[buf]);
      }
      if (!ok) {
        // Wait (bounded) for every MMA already issued before TMEM is released.
        volatile int no_abort = 0;
        Ctl drain{p.status, kDrainLimit, &no_abort, 0u};
        if (PAIR) umma_commit_pair(drain_bar, 0x1);
        else umma_commit(drain_bar);
        wait_bar(drain_bar, 0, drain);
      }
    }
    __syncwarp();
  } else if (XF && warp >= 6) {
    // ------------------------------------------------------------ operand transform
    // Warp xw of the four scales rows 32 xw .. 32 xw + 31 of this CTA's A stage
    // (logit rows m0 + xt), lane = row, with the row's scale for the stage's
    // 256-column tile kept in a register and loaded one tile (4 stages) ahead.
    // The rows written are read only by this CTA's tensor core (each CTA of a
    // pair supplies its own 128 rows of A), so the proxy fence and a CTA-scope
    // arrival order them before the leader issues the MMAs.  With p.xf_store,
    // the unit of output column tile xw mod tiles_n also stores the warp's 32
    // formed rows to the dS chunk (so every row is stored once and the stores
    // spread over the column tiles); a stored stage is released for refilling
    // one stage later, once its store has read it.
    const int xw = warp - 6;
    const int xt = xw * 32 + lane;  // 0 .. 127
    uint32_t n = 0;
    bool ok = true;
    int pend = -1;  // stage whose store may still be reading it (lane 0)
    // the dS chunk is read back only by the next kernel: keep it from evicting
    // the e and W tiles that this kernel's other column tiles re-read from L2
    const uint64_t ds_policy = l2_policy_evict_first();
    for (int t = unit; t < total_tiles && ok; t += units) {
      const UnitRange ur = unit_range(t, p);
      int tm, tn;
      tile_coords(ur.tile, p, tm, tn);
      const int m0 = tm * kBM * kCtas + static_cast<int>(rank) * kBM;
      const int row = m0 + xt;
      const bool live = row < p.xf_rows;
      const bool store =
          p.xf_store != 0 && tn == xw % p.tiles_n && m0 + xw * 32 < p.xf_rows;
      int cur_t = -1, nxt_t = -1;
      float cur = 0.f, nxt = 0.f;
      for (int kb = ur.kb0; kb < ur.kb1; ++kb, ++n) {
        const uint32_t s = n % kNS;
        const uint32_t ph = (n / kNS) & 1u;
        const int k0 = kb * kBKe;
        if (live && (k0 >> 8) != cur_t) {  // entering a new 256-column tile
          cur_t = k0 >> 8;
          cur = (nxt_t == cur_t) ? nxt : __ldg(p.xf_sc + static_cast<int64_t>(cur_t) * p.xf_ld + row);
          nxt_t = cur_t + 1;
          if (nxt_t * 256 < p.num_kb * kBKe)  // prefetch the next tile's scale
            nxt = __ldg(p.xf_sc + static_cast<int64_t>(nxt_t) * p.xf_ld + row);
        }
        if (!wait_bar(&full_bar[s], ph, ctl, true)) {
          ok = false;
          break;
        }
        uint8_t* rows = smem + s * kSBytes + xw * 32 * kRowBytes;  // this warp's 4 KB
        if (live) xf_row(rows + lane * kRowBytes, lane & 7, __float2bfloat162_rn(cur));
        fence_proxy_async_smem();  // generic writes -> the tensor core's and TMA's reads
        __syncwarp();
        if (lane == 0) {
          if (store) {
            tma_store_2d_hint(&tmD, rows, k0, m0 + xw * 32, ds_policy);
            bulk_commit();
          }
          mbar_arrive_cluster(mapa_shared(&ready_bar[s], 0));
          if (pend >= 0) {  // the previous stored stage: its store has read it
            if (store) bulk_wait_read_1();
            else bulk_wait_read_0();
            mbar_arrive(&empty_bar[pend]);
            pend = -1;
          }
          if (store) pend = static_cast<int>(s);
          else mbar_arrive(&empty_bar[s]);
        }
      }
    }
    if (lane == 0) {
      if (ok && pend >= 0) {
        bulk_wait_read_0();
        mbar_arrive(&empty_bar[pend]);
      }
      bulk_wait_all();  // the dS stores have landed before exit
    }
    __syncwarp();
  } else if (warp < 4 || (EG == 2 && warp >= 6)) {
    // ------------------------------------------------------------ epilogue
    // Each warp stages its 32 rows x 32 columns of output in shared memory
    // (two buffers, swizzled to match the output map) and one lane issues a TMA
    // bulk store -- an fp32 add-reduction into global memory when accumulating.
    // A warp reads the TMEM lanes of its quadrant (warp mod 4); with EG = 2,
    // warps 6-9 form group 1 and cover the quadrants 2, 3, 0, 1.
    const int quad = warp & 3;
    const int group = warp < 4 ? 0 : 1;
    constexpr int kBoxStride = EG == 2 ? kStageOutBytes / 2 : kStageOutBytes;  // bf16 only
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* stg = staging + (warp < 4 ? warp : warp - 2) * 2 * kBoxStride;
    const uint64_t out_policy = l2_policy_evict_first();
    uint32_t nbox = 0;  // output boxes this warp has staged
    uint32_t local = 0;
    // The accumulator stage is released with one arrival per warp on the
    // leader CTA's barrier (a remote arrive from the peer CTA of a pair).
    const uint32_t tempty_cluster0 = PAIR ? mapa_shared(&tempty_bar[0], 0) : 0u;
    const uint32_t tempty_cluster1 = PAIR ? mapa_shared(&tempty_bar[1], 0) : 0u;
    auto release = [&](uint32_t buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(buf ? tempty_cluster1 : tempty_cluster0);
        else mbar_arrive(&tempty_bar[buf]);
      }
    };
    // Stage v * scale - shift (32 values of this thread's row) and store the
    // warp's box at output column x, output-map row y (rows past the map's
    // extent are not written).  issue is false (uniformly over the warp) when
    // all of the warp's rows lie past the output's extent: then nothing is
    // staged either.  Each staged box commits exactly one bulk group, which is
    // what lets the wait below (at most one group still reading) prove that
    // the store which last used this buffer, two boxes back, has read it.
    auto store_box = [&](const uint32_t(&v)[32], float scale, float shift, int x, int y,
                         bool fp32_out, bool reduce, bool issue) {
      if (!issue) return;
      uint8_t* sb = stg + (nbox & 1u) * kBoxStride;
      ++nbox;
      if (lane == 0) bulk_wait_read_1();  // the store that last used sb has read it
      __syncwarp();
      if (fp32_out) {  // 128-byte rows, 128-byte swizzle: chunk j at j ^ (row & 7)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 q = make_float4(fmaf(__uint_as_float(v[4 * j]), scale, -shift),
                                       fmaf(__uint_as_float(v[4 * j + 1]), scale, -shift),
                                       fmaf(__uint_as_float(v[4 * j + 2]), scale, -shift),
                                       fmaf(__uint_as_float(v[4 * j + 3]), scale, -shift));
          *reinterpret_cast<float4*>(sb + lane * 128 + ((j ^ (lane & 7)) << 4)) = q;
        }
      } else {  // bf16: 64-byte rows, 64-byte swizzle: chunk j at j ^ ((row >> 1) & 3)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = fmaf(__uint_as_float(v[8 * j + i]), scale, -shift);
          store_vec<__nv_bfloat16>(
              reinterpret_cast<__nv_bfloat16*>(sb + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)),
              f);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // outputs are streamed, never re-read by this kernel: evict them from
        // L2 first so the operand tiles that other tiles share stay resident
        if (reduce) tma_reduce_add_2d_hint(&tmC, sb, x, y, out_policy);
        else tma_store_2d_hint(&tmC, sb, x, y, out_policy);
        bulk_commit();
      }
    };
    constexpr bool kElemF32 = sizeof(Elem) == 4;
    for (int t = unit; t < total_tiles; t += units, ++local) {
      // EG = 2: group g takes the units whose accumulator is buffer g
      if (EG == 2 && static_cast<int>(local & 1u) != group) continue;
      const UnitRange ur = unit_range(t, p);
      int tm, tn;
      tile_coords(ur.tile, p, tm, tn);
      const uint32_t buf = local % kAccBufs;
      const uint32_t aph = (local / kAccBufs) & 1u;
      if (!wait_bar(&tfull_bar[buf], aph, ctl, kPark)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_base + buf * kBN;
      const int row0 = tm * kBM * kCtas + static_cast<int>(rank) * kBM + quad * 32;
      const int grow = row0 + lane;
      const bool rv = grow < p.rows_valid;
      const bool warp_rows = row0 < p.rows_valid;  // any row of this warp's box exists
      const int col0 = tn * kTileN;

      if (EPI == EPI_STATS) {
        const float rscale = (p.T_row != nullptr && rv) ? 1.f / p.T_row[grow] : p.scale;
        const float s2 = rscale * kLog2e;
        float mx = -INFINITY, se = 0.f, cross = 0.f;
        int gi = 0, gcol = 0x7fffffff;
        const int* ri = nullptr;
        const float* rq = nullptr;
        if (p.ktop > 0 && rv) {
          ri = p.sidx + static_cast<int64_t>(grow) * p.ktop;
          rq = p.sq + static_cast<int64_t>(grow) * p.ktop;
          int lo = 0, hi = p.ktop;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(ri + mid) < col0) lo = mid + 1; else hi = mid;
          }
          gi = lo;
          gcol = gi < p.ktop ? __ldg(ri + gi) : 0x7fffffff;
        }
        // Teacher-hidden student pass (tbuf given): the teacher's stored tile
        // t~ - mt gives, per column, w = 2^((t~ - mt) log2 e) and t~ - s~; the
        // tile's sums A = sum w (t~ - s~) and U = sum 2^(x - max) (s~ - t~) are
        // formed in pass 2 from fp32 values.  The teacher values of a 32-column
        // slab are loaded one slab ahead (slab 0 before pass 1) so that their
        // latency overlaps the work on the previous slab.
        const bool hid = p.tbuf != nullptr && rv;
        const float* trow = hid ? p.tbuf + static_cast<int64_t>(grow) * p.tld : nullptr;
        auto load_t = [&](int cb, float(&tv)[32]) {
          const int nv = p.cols_valid - cb;
          if (nv >= 32) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 t4 = __ldg(reinterpret_cast<const float4*>(trow + cb) + j);
              tv[4 * j] = t4.x;
              tv[4 * j + 1] = t4.y;
              tv[4 * j + 2] = t4.z;
              tv[4 * j + 3] = t4.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) tv[i] = i < nv ? __ldg(trow + cb + i) : 0.f;
          }
        };
        float tcur[32];
        if (hid) load_t(col0, tcur);
        // Pass 1: the row's maximum over this tile (base-2 units) and the
        // cached entries' cross term, from the fp32 accumulator.
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + c * 32, v);
          tmem_ld_wait();
          const int cb = col0 + c * 32;
          const int nvalid = p.cols_valid - cb;  // columns < V in this slab
#pragma unroll
          for (int i = 0; i < 32; ++i)
            mx = fmaxf(mx, i < nvalid ? __uint_as_float(v[i]) * s2 : -INFINITY);
          while (gcol < cb + 32) {  // cached entries inside this 32-column slab
            const int k = gcol - cb;
            float val = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) val = (i == k) ? __uint_as_float(v[i]) : val;
            cross += __ldg(rq + gi) * (val * rscale);
            ++gi;
            gcol = gi < p.ktop ? __ldg(ri + gi) : 0x7fffffff;
          }
        }
        // Pass 2: sum of 2^(x - max) and the stored values.  STORE_SHIFTED
        // stores s~ - max: the entries that carry the probability mass sit near
        // 0, where the stored value's rounding error vanishes; readers add the
        // maximum back from the tile statistics.  STORE_EXP stores the
        // exponentials 2^(x - max) in (0, 1].
        const float mt = hid ? __ldg(&p.tpart[static_cast<int64_t>(grow) * p.tiles_n + tn].x) *
                                   kLn2f
                             : 0.f;
        float A = 0.f, U = 0.f;
        const float shift = (p.partials != nullptr && mx > -INFINITY) ? mx * kLn2f : 0.f;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + c * 32, v);
          tmem_ld_wait();
          if (c == kBN / 32 - 1) release(buf);
          const int cb = col0 + c * 32;
          const int nvalid = p.cols_valid - cb;
          if (nvalid <= 0) continue;
          float e[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            e[i] = i < nvalid ? ex2_approx(fmaf(__uint_as_float(v[i]), s2, -mx)) : 0.f;
            se += e[i];
          }
          if (hid) {
            float tnxt[32];
            const bool more = c + 1 < kBN / 32 && nvalid > 32;
            if (more) load_t(cb + 32, tnxt);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (i < nvalid) {
                const float d = (tcur[i] + mt) - __uint_as_float(v[i]) * rscale;  // t~ - s~
                A = fmaf(ex2_approx(tcur[i] * kLog2e), d, A);
                U = fmaf(e[i], -d, U);
              }
            }
            if (more) {
#pragma unroll
              for (int i = 0; i < 32; ++i) tcur[i] = tnxt[i];
            }
          }
          if (p.store == STORE_SHIFTED) {
            store_box(v, rscale, shift, cb, row0, p.out_f32 != 0, false, warp_rows);
          } else if (p.store == STORE_EXP) {
            uint32_t eb[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) eb[i] = __float_as_uint(e[i]);
            store_box(eb, 1.f, 0.f, cb, row0, false, false, warp_rows);
          }
        }
        if (rv && p.partials != nullptr)
          p.partials[static_cast<int64_t>(grow) * p.tiles_n + tn] =
              p.tbuf != nullptr ? make_float4(mx, se, A, U) : make_float4(mx, se, cross, 0.f);
      } else if (EPI == EPI_DLOGITS) {
        float coef = 0.f, cm = 0.f, l2 = 0.f;
        const float rscale = (p.T_row != nullptr && rv) ? 1.f / p.T_row[grow] : p.scale;
        int gi = 0, gcol = 0x7fffffff;
        const int* ri = nullptr;
        const float* rq = nullptr;
        if (rv) {
          const bool keep = p.mask == nullptr || p.mask[grow] != 0;
          const float g = p.g_dev != nullptr ? *p.g_dev : p.g_host;
          const float n = *p.norm;
          coef = (keep && n > 0.f) ? g / n * rscale : 0.f;
          cm = coef * p.rowinfo[grow].x;
          l2 = p.lse[grow] * kLog2e;
          ri = p.sidx + static_cast<int64_t>(grow) * p.ktop;
          rq = p.sq + static_cast<int64_t>(grow) * p.ktop;
          int lo = 0, hi = p.ktop;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(ri + mid) < col0) lo = mid + 1; else hi = mid;
          }
          gi = lo;
          gcol = gi < p.ktop ? __ldg(ri + gi) : 0x7fffffff;
        }
        const float s2 = rscale * kLog2e;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + c * 32, v);
          tmem_ld_wait();
          if (c == kBN / 32 - 1) release(buf);
          const int cb = col0 + c * 32;
          if (cb >= p.cols_valid) continue;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = __uint_as_float(v[i]) * s2;
            v[i] = __float_as_uint(cm * ex2_approx(x - l2));
          }
          while (gcol < cb + 32) {  // subtract c q at the cached ids inside this slab
            const int k = gcol - cb;
            const float cq = coef * __ldg(rq + gi);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = (i == k) ? __float_as_uint(__uint_as_float(v[i]) - cq) : v[i];
            ++gi;
            gcol = gi < p.ktop ? __ldg(ri + gi) : 0x7fffffff;
          }
          if (sizeof(Elem) == 4) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(round_tf32_dev(__uint_as_float(v[i])));
          }
          store_box(v, 1.f, 0.f, cb, row0, kElemF32, false, warp_rows);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kTileN / 32; ++c) {  // both halves: TMEM columns are contiguous
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + c * 32, v);
          tmem_ld_wait();
          if (c == kTileN / 32 - 1) release(buf);
          const int cb = col0 + c * 32;
          if (cb >= p.cols_valid) continue;
          if (EPI == EPI_STORE)
            store_box(v, 1.f, 0.f, cb, row0, kElemF32, false, warp_rows);
          else  // EPI_ACCUM, fp32 out; K-part ks writes its own block of output rows
            store_box(v, 1.f, 0.f, cb, row0 + ur.ks * p.split_rows, true, p.beta != 0, warp_rows);
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // every output box has landed before exit
    __syncwarp();
  }

  // Every role of both CTAs has finished (or given up).  After an abort, copies
  // that were issued but never consumed may still be in flight; wait for them
  // before either CTA of the pair can exit.
  __syncthreads();
  if (PAIR) cluster_sync();
  bool aborted = *abort_flag != 0;
  if (PAIR) aborted = aborted || ld_cluster_u32(peer_abort) != 0u;
  if (aborted && warp == 4 && lane == 0) {
    volatile int no_abort = 0;
    const Ctl drain{p.status, kDrainLimit, &no_abort, 0u};
    const uint32_t mine = *issued_slot;
    uint32_t hi = mine;
    bool drain_here = true;
    if (!kLocalCopies) {
      // Both CTAs' copies complete on the leader's barriers, which the leader
      // armed for both CTAs' bytes of every stage it issued.  Settle the stages
      // one producer issued and the other did not, then wait for the last ring's
      // worth of stages.
      drain_here = leader;
      if (leader) {
        const uint32_t peer = ld_cluster_u32(mapa_shared(issued_slot, 1));
        for (uint32_t n = peer; n < mine; ++n)  // the peer's bytes never come
          mbar_complete_tx(&full_bar[n % kNS], kSBytes);
        for (uint32_t n = mine; n < peer; ++n)  // armed for the peer's bytes only
          mbar_arrive_expect_tx(&full_bar[n % kNS], kSBytes);
        hi = peer > mine ? peer : mine;
      }
    }
    if (drain_here) {
      const uint32_t first = hi > kNS ? hi - kNS : 0;
      for (uint32_t n = first; n < hi; ++n) wait_bar(&full_bar[n % kNS], (n / kNS) & 1u, drain);
    }
  }
  __syncthreads();
  if (PAIR) cluster_sync();  // neither CTA of a pair leaves while the other still works
  if (warp == 5) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace ckl
