// Tensor-core GEMM for sm_100a: C = A B^T with bf16 (or fp16) operands and
// fp32 accumulation. Each operand is K-major (A as M x K rows, B as N x K) or
// MN-major (A stored as K x M rows, B as K x N), read as stored by TMA.
//
// Persistent, warp-specialised CTA (one per SM): warp 0 issues TMA tile loads
// into a 4-stage shared-memory ring, warp 1 issues tcgen05.mma (128 x 256 x 16)
// into one of two TMEM accumulators, warps 2-5 drain the other accumulator
// with tcgen05.ld and run the epilogue, so the epilogue of tile i overlaps
// the MMAs of tile i+1. Every mbarrier wait is bounded in time: on expiry the
// CTA raises the timeout bit of the device status word, drains its own
// copies and MMAs (bounded again), frees its TMEM and returns.
#include <cfloat>
#include <cstring>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "tc_ptx.cuh"

namespace dust {
namespace {

// BM rows of A and BN accumulator columns per CTA; BK-deep stages.
constexpr int BM = 128, BN = 256, BK = 64;
static_assert(BN == kTcTileN, "reward partials are laid out per BN-column tile");
constexpr int TMEM_COLS = 2 * BN;
// warp 0: TMA producer; warp 1: MMA issuer; warps 2..9: epilogue, two per
// TMEM lane quarter, each draining one half of the accumulator's columns
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int HALF_N = BN / 2;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// Reward epilogue: each epilogue warp stages the probability rows of the (at
// most two) tokens its 32 rows belong to, over its HALF_N columns, per
// accumulator.
constexpr int PSTAGE_FLOATS = 2 * HALF_N;
constexpr size_t PSTAGE_BYTES = (size_t)EPI_WARPS * 2 * PSTAGE_FLOATS * 4;
constexpr int kMaxStages = 6;
// An MN-major operand tile: boxes of 64 MN elements x BK rows of K.
constexpr uint32_t MN_BOX = 64 * BK * 2;

// The fp32 store of kEpiF32Lse goes through shared memory: each epilogue
// warp writes its 32 rows x 32 columns into one of STORE_BUFS 4 KB boxes
// (128-byte swizzled, so the row-per-thread writes hit distinct banks) and
// one lane stores the box by TMA, instead of every thread writing 16 bytes
// into each of 32 rows per instruction.
constexpr int STORE_BOX = 32;
constexpr int STORE_BOX_BYTES = STORE_BOX * STORE_BOX * 4;
constexpr int STORE_BUFS = 1;
constexpr size_t STORE_BYTES = (size_t)EPI_WARPS * STORE_BUFS * STORE_BOX_BYTES;

// Single CTA: a 128 x 256 tile per SM, A and all 256 rows of B staged by the
// CTA (48 KB per 64-deep stage, 4 stages). CTA pair (cta_group::2): a
// 256 x 256 tile per pair of SMs; each CTA stages its 128 rows of A and 128
// of the 256 rows of B (32 KB per stage, 6 stages) and the leader's MMAs read
// both CTAs' shared memory, so every SM is fed a third fewer bytes per flop.
// kEpiF32Lse gives up one operand stage per 32 KB of store boxes.
template <bool PAIR, int KIND>
struct Cfg {
  static constexpr bool STORE = KIND == kEpiF32Lse;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;
  static constexpr int STAGES = PAIR ? (STORE ? 6 - STORE_BUFS : 6) : (STORE ? 5 - STORE_BUFS : 4);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  // after the stages (1024-byte aligned): the store boxes or the reward's
  // probability staging, then the barrier block
  static constexpr size_t EXTRA = STORE ? STORE_BYTES : PSTAGE_BYTES;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EXTRA + 256;
  static_assert(STAGES <= kMaxStages, "barrier arrays");
  static_assert(EXTRA % 1024 == 0 && STAGE_BYTES % 1024 == 0, "swizzled boxes need 1024-byte alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct TcParams {
  int64_t M, N, K;
  int m_tiles, n_tiles, num_kb;  // m_tiles counts Cfg::TILE_M-row tiles
  int tma_store;                 // kEpiF32Lse: C is stored through tmC
  int a_mn, b_mn;                // operand stored MN-major (K x M, K x N rows)
  int f16;                       // fp16 operands (kind::f16 takes both types)
  EpiDesc e;
  uint32_t* status;
  uint64_t wait_ns;  // limit of the pipeline waits (teardown waits keep kWaitLimitNs)
};

struct Shared {
  uint64_t full[kMaxStages], empty[kMaxStages], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Shared) <= 256, "barrier block overlaps the staging area");

// Wait for phase `parity` of an mbarrier for at most limit_ns (0: a single
// poll). On expiry the CTA's abort flag and the timeout bit of the status word
// are set and false returns; a raised abort flag (checked every 64 polls)
// also ends the wait.
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* status,
                             uint64_t limit_ns = kWaitLimitNs) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  if (limit_ns == 0) {
    *abort = 1;
    atomicOr(status, kStatusTimeout);
    return false;
  }
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (ptx::globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Epilogue of 32 consecutive columns [n, n+32) of row m (output row mo).
template <int KIND>
__device__ __forceinline__ void epilogue32(const TcParams& p, int64_t m, int64_t mo, int64_t n,
                                           float* v, float escale) {
  const EpiDesc& e = p.e;
  const bool full = n + 32 <= p.N;
  if (KIND == kEpiF32) {
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] *= escale;
  }
  if (KIND == kEpiF32 || KIND == kEpiF32Lse || KIND == kEpiGeluSplit) {
    float* dst = e.C + (KIND == kEpiF32 ? mo : m) * e.ldc + n;
    if (full && ((e.ldc & 3) == 0) && (((uintptr_t)e.C & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (n + q < p.N) dst[q] = v[q];
    }
  }
  if (KIND == kEpiBF16) {
    __nv_bfloat16* dst = e.Cb + m * e.ldcb + n;
    if (full && ((e.ldcb & 7) == 0) && (((uintptr_t)e.Cb & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[8 * q + 0], v[8 * q + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
        uint4 u;
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        reinterpret_cast<uint4*>(dst)[q] = u;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (n + q < p.N) dst[q] = __float2bfloat16_rn(v[q]);
    }
  }
  if (KIND == kEpiGeluSplit) {
    __nv_bfloat16* hi = e.Cb + m * e.ldcb + n;
    __nv_bfloat16* lo = hi + e.split;
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (n + q < p.N) split_bf16(gelu64((double)v[q]), hi + q, lo + q);
  }
  if (KIND == kEpiResidSplit) {
    // h = resid (+ its lo plane) + acc in fp32 (error 2^-24 relative), then
    // the 2^-17 hi/lo split; 16-byte loads and stores when the row is aligned
    __nv_bfloat16* hi = e.Cb + m * e.ldcb + n;
    __nv_bfloat16* lo = hi + e.split;
    const __nv_bfloat16* r = (const __nv_bfloat16*)e.resid + m * e.ldr + n;
    const __nv_bfloat16* r2 = e.rsplit > 0 ? r + e.rsplit : nullptr;
    const bool vec = full && ((e.ldcb | e.split | e.ldr | e.rsplit) & 7) == 0 &&
                     (((uintptr_t)e.Cb | (uintptr_t)e.resid) & 15) == 0;
    if (vec) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 ra = reinterpret_cast<const uint4*>(r)[q];
        const uint4 rb = r2 ? reinterpret_cast<const uint4*>(r2)[q] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 pa = *reinterpret_cast<const __nv_bfloat162*>(&wa[h]);
          const __nv_bfloat162 pb = *reinterpret_cast<const __nv_bfloat162*>(&wb[h]);
          const float x0 = __low2float(pa) + __low2float(pb) + v[8 * q + 2 * h];
          const float x1 = __high2float(pa) + __high2float(pb) + v[8 * q + 2 * h + 1];
          const __nv_bfloat162 hh = __floats2bfloat162_rn(x0, x1);
          const __nv_bfloat162 ll = __floats2bfloat162_rn(x0 - __low2float(hh), x1 - __high2float(hh));
          hw[h] = *reinterpret_cast<const uint32_t*>(&hh);
          lw[h] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        reinterpret_cast<uint4*>(hi)[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        reinterpret_cast<uint4*>(lo)[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        if (n + q < p.N) {
          float x = __bfloat162float(r[q]) + v[q];
          if (r2) x += __bfloat162float(r2[q]);
          split_bf16(x, hi + q, lo + q);
        }
      }
    }
  }
  if (KIND == kEpiSplit) {
    __nv_bfloat16* hi = e.Cb + m * e.ldcb + n;
    __nv_bfloat16* lo = hi + e.split;
    if (full && ((e.ldcb & 7) == 0) && ((e.split & 7) == 0) && (((uintptr_t)e.Cb & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float a = v[8 * q + 2 * h], b = v[8 * q + 2 * h + 1];
          const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
          const __nv_bfloat162 ll = __floats2bfloat162_rn(a - __low2float(hh), b - __high2float(hh));
          hw[h] = *reinterpret_cast<const uint32_t*>(&hh);
          lw[h] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        reinterpret_cast<uint4*>(hi)[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        reinterpret_cast<uint4*>(lo)[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (n + q < p.N) split_bf16(v[q], hi + q, lo + q);
    }
  }
}

// Online softmax partial of a row over 32 more columns [n, n+32): the running
// maximum and the sum of exponentials relative to it, as 4 independent chains.
__device__ __forceinline__ void lse_chunk(const TcParams& p, int64_t n, const float* v, float& rmax,
                                          float& rsum) {
  float cm[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
  for (int q = 0; q < 32; ++q)
    if (n + q < p.N) cm[q & 3] = fmaxf(cm[q & 3], v[q]);
  const float nm = fmaxf(rmax, fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3])));
  float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int q = 0; q < 32; ++q)
    if (n + q < p.N) cs[q & 3] += __expf(v[q] - nm);
  rsum = fmaf(rsum, __expf(rmax - nm), (cs[0] + cs[1]) + (cs[2] + cs[3]));
  rmax = nm;
}

// Tile order: bands of kGroupM M-tiles swept across all N-tiles, M fastest
// within the band. The CTAs running at the same time then cover a compact
// kGroupM x (SMs / kGroupM) block of tiles, so the band of A (kGroupM * 128
// rows) and the current few B tiles stay in L2; A is read from HBM once and B
// once per band.
constexpr int kGroupM = 16;

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int* m_blk,
                                            int* n_blk) {
  const int band = tile / (kGroupM * n_tiles);
  const int r = tile - band * (kGroupM * n_tiles);
  const int rows = min(kGroupM, m_tiles - band * kGroupM);
  *m_blk = band * kGroupM + r % rows;
  *n_blk = r / rows;
}

// expm1 of a perturbed logit without a branch: degree-5 Taylor polynomial
// below 1/16 (relative truncation < 2e-9); above, e^x - 1 from the hardware
// exponential, whose few-ulp error on e^x is below 1e-5 relative to
// expm1(x) >= 0.06 there (the reward needs sum_n p_n expm1 to ~1e-7 absolute).
__device__ __forceinline__ float expm1_guarded(float x) {
  float q = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
  q = fmaf(x, q, 1.0f / 6.0f);
  q = fmaf(x, q, 0.5f);
  q = fmaf(x, q, 1.0f);
  const float big = __expf(x) - 1.0f;
  return fabsf(x) < 0.0625f ? x * q : big;
}

// Reward epilogue of 32 columns of row m (target column yt): returns
// sum_n P[t, n] expm1(dz_n) and records dz at the target column. prow points
// at P[t, n]: a staged shared-memory copy (zero past column N) when `staged`,
// else the row in global memory.
// The degree-5 series of expm1_guarded for a pair, in packed fp32x2
// arithmetic (each lane rounds as the scalar form does).
__device__ __forceinline__ float2 expm1_series5_x2(float2 x) {
  float2 q = __ffma2_rn(x, make_float2(1.0f / 120.0f, 1.0f / 120.0f),
                        make_float2(1.0f / 24.0f, 1.0f / 24.0f));
  q = __ffma2_rn(x, q, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
  q = __ffma2_rn(x, q, make_float2(0.5f, 0.5f));
  q = __ffma2_rn(x, q, make_float2(1.0f, 1.0f));
  return __fmul2_rn(x, q);
}

__device__ __forceinline__ float reward32(const TcParams& p, int64_t m, int32_t yt, int64_t n,
                                          const float* prow, bool staged, const float* v) {
  // four independent sums, so the adds do not form one 32-long chain
  float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
  float amax = 0.0f;
#pragma unroll
  for (int q = 0; q < 32; ++q) amax = fmaxf(amax, fabsf(v[q]));
  if (amax < 0.0625f && (staged || (n + 32 <= p.N && (p.N & 3) == 0))) {
    // every |dz| of the lane's 32 columns in the series' range (the usual
    // case): the series alone, two columns per packed operation
    float2 sa = make_float2(0.0f, 0.0f), sb = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 pv = staged ? reinterpret_cast<const float4*>(prow)[q]
                               : __ldg(reinterpret_cast<const float4*>(prow) + q);
      sa = __ffma2_rn(make_float2(pv.x, pv.y),
                      expm1_series5_x2(make_float2(v[4 * q + 0], v[4 * q + 1])), sa);
      sb = __ffma2_rn(make_float2(pv.z, pv.w),
                      expm1_series5_x2(make_float2(v[4 * q + 2], v[4 * q + 3])), sb);
    }
    s0 = sa.x;
    s1 = sa.y;
    s2 = sb.x;
    s3 = sb.y;
  } else if (staged || (n + 32 <= p.N && (p.N & 3) == 0)) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 pv = staged ? reinterpret_cast<const float4*>(prow)[q]
                               : __ldg(reinterpret_cast<const float4*>(prow) + q);
      s0 = fmaf(pv.x, expm1_guarded(v[4 * q + 0]), s0);
      s1 = fmaf(pv.y, expm1_guarded(v[4 * q + 1]), s1);
      s2 = fmaf(pv.z, expm1_guarded(v[4 * q + 2]), s2);
      s3 = fmaf(pv.w, expm1_guarded(v[4 * q + 3]), s3);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (n + q < p.N) s0 = fmaf(prow[q], expm1_guarded(v[q]), s0);
  }
  const float s = (s0 + s1) + (s2 + s3);
  if (yt >= n && yt < n + 32) {
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (n + q == yt) p.e.dzy[m] = v[q];
  }
  return s;
}

template <int KIND, bool PAIR>
__global__ __launch_bounds__(THREADS, 1) void k_gemm_tc(const __grid_constant__ CUtensorMap tmA,
                                                        const __grid_constant__ CUtensorMap tmB,
                                                        const __grid_constant__ CUtensorMap tmC,
                                                        TcParams p) {
  using C = Cfg<PAIR, KIND>;
  constexpr int STAGES = C::STAGES, A_BYTES = C::A_BYTES, B_BYTES = C::B_BYTES;
  constexpr int STAGE_BYTES = C::STAGE_BYTES, TILE_M = C::TILE_M;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* basep = smem_raw + (base - raw);
  const uint32_t sA = base;                           // STAGES x A tile
  const uint32_t sB = base + STAGES * A_BYTES;        // STAGES x B tile
  float* pstage = reinterpret_cast<float*>(basep + STAGES * STAGE_BYTES);
  const uint32_t sStore = base + STAGES * STAGE_BYTES;  // kEpiF32Lse store boxes
  Shared* sh = reinterpret_cast<Shared*>(basep + STAGES * STAGE_BYTES + C::EXTRA);
  volatile int* abort = &sh->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.m_tiles * p.n_tiles;
  // MN-major and fp16 operands are taken by the plain fp32 epilogue (the
  // weight gradient) only; the other kinds keep the K-major bf16 code
  const bool a_mn = KIND == kEpiF32 && p.a_mn != 0;
  const bool b_mn = KIND == kEpiF32 && p.b_mn != 0;
  const bool f16 = KIND == kEpiF32 && p.f16 != 0;
  // CTA pairs work on one tile together: unit = pair index, rank 0 leads
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(ptx::smem_u32(&sh->full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&sh->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(ptx::smem_u32(&sh->tfull[a]), 1);
      // the leader's MMAs wait for the epilogue warps of both CTAs
      ptx::mbar_init(ptx::smem_u32(&sh->tempty[a]), PAIR ? 2 * EPI_WARPS : EPI_WARPS);
    }
    ptx::mbar_init(ptx::smem_u32(&sh->drain), 1);
    sh->abort = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
    ptx::prefetch_map(&tmA);
    ptx::prefetch_map(&tmB);
    if (C::STORE && p.tma_store) ptx::prefetch_map(&tmC);
  }
  if (warp == 1) {
    if (PAIR) {
      ptx::tmem_alloc_pair(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  ptx::tc_fence_before();
  // both CTAs' barriers and TMEM exist before either signals the other
  if (PAIR) ptx::cluster_sync(); else __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // bit s: stage s holds a copy / its parity
      for (int tile = unit0; tile < total && !*abort; tile += units) {
        int m_blk, n_blk;
        tile_coords(tile, p.m_tiles, p.n_tiles, &m_blk, &n_blk);
        const int a_row = m_blk * TILE_M + (int)rank * BM;
        const int b_row = n_blk * BN + (int)rank * C::B_ROWS;
        // a K-major operand tile is one box of rows x 64 K; an MN-major one
        // is rows / 64 boxes of 64 MN x 64 K rows, MN_BOX bytes apart
        auto load = [&](uint32_t dst, const CUtensorMap* map, bool mn, int rows, int r0, int k0,
                        uint32_t bar) {
          if (!mn) {
            if (PAIR) ptx::tma_load_2d_pair(dst, map, k0, r0, bar);
            else ptx::tma_load_2d(dst, map, k0, r0, bar);
            return;
          }
          for (int j = 0; j < rows / 64; ++j) {
            if (PAIR) ptx::tma_load_2d_pair(dst + j * MN_BOX, map, r0 + 64 * j, k0, bar);
            else ptx::tma_load_2d(dst + j * MN_BOX, map, r0 + 64 * j, k0, bar);
          }
        };
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&sh->empty[stage]), phase ^ 1u, abort, p.status, p.wait_ns)) break;
          const uint32_t fb = ptx::smem_u32(&sh->full[stage]);
          uint32_t bar = fb;
          if (PAIR) {
            // both CTAs' bytes complete on the leader's barrier
            if (leader) ptx::mbar_expect_tx(fb, 2 * STAGE_BYTES);
            bar = ptx::mapa_shared(fb, 0);
          } else {
            ptx::mbar_expect_tx(fb, STAGE_BYTES);
          }
          load(sA + stage * A_BYTES, &tmA, a_mn, BM, a_row, kb * BK, bar);
          load(sB + stage * B_BYTES, &tmB, b_mn, C::B_ROWS, b_row, kb * BK, bar);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy this thread issued has landed before the CTA can exit: a
      // single CTA (or the leader) sees its stages complete; the pair's
      // second CTA sees them consumed (the MMAs waited for their bytes)
      int dummy = 0;
      for (int s = 0; s < STAGES; ++s)
        if ((armed >> s) & 1u) {
          if (PAIR && !leader)
            wait_bounded(ptx::smem_u32(&sh->empty[s]), (armed_parity >> s) & 1u, &dummy, p.status);
          else
            wait_bounded(ptx::smem_u32(&sh->full[s]), (armed_parity >> s) & 1u, &dummy, p.status);
        }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && leader) {
      const uint32_t idesc =
          (f16 ? ptx::idesc_f16_f32(TILE_M, BN) : ptx::idesc_bf16_f32(TILE_M, BN)) |
          (a_mn ? ptx::kIdescAMn : 0u) | (b_mn ? ptx::kIdescBMn : 0u);
      // per 16-deep MMA step: 32 bytes along a K-major row, two 8-row
      // swizzle atoms (2048 bytes) down an MN-major tile
      const uint32_t a_step = a_mn ? 2048u : 32u, b_step = b_mn ? 2048u : 32u;
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool issued = false;
      for (int tile = unit0; tile < total && !*abort; tile += units, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&sh->tempty[acc]), acc_phase ^ 1u, abort, p.status, p.wait_ns)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&sh->full[stage]), phase, abort, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sA + stage * A_BYTES, b0 = sB + stage * B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t ak = a0 + k * a_step, bk = b0 + k * b_step;
            const uint64_t ad = a_mn ? ptx::sdesc_mnmajor_sw128(ak, MN_BOX) : ptx::sdesc_kmajor_sw128(ak);
            const uint64_t bd = b_mn ? ptx::sdesc_mnmajor_sw128(bk, MN_BOX) : ptx::sdesc_kmajor_sw128(bk);
            if (PAIR)
              ptx::mma_f16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0);
            else
              ptx::mma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          issued = true;
          if (PAIR)
            ptx::mma_commit_pair(ptx::smem_u32(&sh->empty[stage]), 0x3);
          else
            ptx::mma_commit(ptx::smem_u32(&sh->empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR)
          ptx::mma_commit_pair(ptx::smem_u32(&sh->tfull[acc]), 0x3);
        else
          ptx::mma_commit(ptx::smem_u32(&sh->tfull[acc]));
      }
      if (issued) {
        // all MMAs complete before TMEM is released (in both CTAs of a pair)
        if (PAIR)
          ptx::mma_commit_pair(ptx::smem_u32(&sh->drain), 0x3);
        else
          ptx::mma_commit(ptx::smem_u32(&sh->drain));
        int dummy = 0;
        wait_bounded(ptx::smem_u32(&sh->drain), 0, &dummy, p.status);
      }
    } else if (PAIR && lane == 0 && unit0 < total) {
      // the second CTA of a pair: the leader's MMAs write this CTA's TMEM too
      int dummy = 0;
      wait_bounded(ptx::smem_u32(&sh->drain), 0, &dummy, p.status);
    }
  } else {
    // ---------------- epilogue warps 2..9 ----------------
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
    const int row = quad * 32 + lane;
    const int half = (warp - 2) >> 2;  // columns [HALF_N half, HALF_N (half + 1)) of the tile
    int it = 0;
    // kEpiF32: the output scale (a power of two the operands' producer wrote)
    const float escale = (KIND == kEpiF32 && p.e.scale) ? *p.e.scale : 1.0f;
    int nbox = 0;  // kEpiF32Lse: store boxes this warp has issued
    const uint32_t box0 = sStore + (uint32_t)((warp - 2) * STORE_BUFS * STORE_BOX_BYTES);
    const uint32_t tempty0 =
        PAIR ? ptx::mapa_shared(ptx::smem_u32(&sh->tempty[0]), 0) : ptx::smem_u32(&sh->tempty[0]);
    const uint32_t tempty1 =
        PAIR ? ptx::mapa_shared(ptx::smem_u32(&sh->tempty[1]), 0) : ptx::smem_u32(&sh->tempty[1]);
    for (int tile = unit0; tile < total; tile += units, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
      int m_blk, n_blk;
      tile_coords(tile, p.m_tiles, p.n_tiles, &m_blk, &n_blk);
      // Reward: stage P[t, n-tile] of this warp's tokens while the tile's MMAs
      // run (each row otherwise waits on its own global loads chunk by chunk).
      bool staged = false;
      int64_t t_first = 0;
      float* stg = pstage + ((warp - 2) * 2 + acc) * PSTAGE_FLOATS;
      if (KIND == kEpiReward) {
        const int64_t m_first = (int64_t)m_blk * TILE_M + (int64_t)rank * BM + quad * 32;
        if (m_first < p.M && (p.N & 3) == 0) {
          const int64_t m_last = min(m_first + 31, p.M - 1);
          t_first = p.e.t0 + m_first / p.e.draws;
          const int64_t t_last = p.e.t0 + m_last / p.e.draws;
          staged = t_last - t_first <= 1;
          if (staged) {
            float4 pv[PSTAGE_FLOATS / 128];
#pragma unroll
            for (int j = 0; j < PSTAGE_FLOATS / 128; ++j) {
              // float4 index q: token q / (HALF_N/4), column 4 (q % (HALF_N/4)) of the half
              const int q = lane + 32 * j;
              const int64_t t = t_first + q / (HALF_N / 4);
              const int64_t n = (int64_t)n_blk * BN + half * HALF_N + 4 * (q % (HALF_N / 4));
              pv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (t <= t_last && n < p.N)
                pv[j] = __ldg(reinterpret_cast<const float4*>(p.e.P + t * p.N + n));
            }
            __syncwarp();  // the previous tile that used this buffer is done
#pragma unroll
            for (int j = 0; j < PSTAGE_FLOATS / 128; ++j)
              reinterpret_cast<float4*>(stg)[lane + 32 * j] = pv[j];
            __syncwarp();
          }
        }
      }
      if (!wait_bounded(ptx::smem_u32(&sh->tfull[acc]), acc_phase, abort, p.status, p.wait_ns)) break;
      ptx::tc_fence_after();
      const int64_t m = (int64_t)m_blk * TILE_M + (int64_t)rank * BM + row;
      int64_t mo = m;
      if (p.e.c_row_mul != 0 && m < p.M)
        mo = (int64_t)(((unsigned long long)m * (unsigned long long)p.e.c_row_mul) %
                       (unsigned long long)p.M);
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      int64_t t_row = 0;
      int32_t yt = 0;
      if (KIND == kEpiReward && m < p.M) {
        t_row = p.e.t0 + m / p.e.draws;
        yt = p.e.y[t_row];
        if (yt < 0 || (int64_t)yt >= p.N) yt = 0;  // reported by the loss kernel
      }
      float s_row = 0.0f;
      float rmax = -FLT_MAX, rsum = 0.0f;  // kEpiF32Lse: online softmax partial of the row
#pragma unroll 1
      for (int c = half * (HALF_N / 32); c < (half + 1) * (HALF_N / 32); ++c) {
        const int64_t n = (int64_t)n_blk * BN + c * 32;
        float v[32];
        ptx::tmem_ld32(taddr + (uint32_t)(c * 32), v);
        if (KIND == kEpiReward) {
          if (m < p.M && n < p.N) {
            const float* prow = staged ? stg + (t_row - t_first) * HALF_N + (c * 32 - half * HALF_N)
                                       : p.e.P + t_row * p.N + n;
            s_row += reward32(p, m, yt, n, prow, staged, v);
          }
        } else if (C::STORE && p.tma_store && n < p.N) {
          // this warp's 32 x 32 box: row `lane` at byte 128 lane, its 16-byte
          // chunk q at position q ^ (lane & 7) (the 128-byte swizzle of tmC);
          // the box's previous store from this buffer has read it by now
          const uint32_t box = box0 + (uint32_t)((nbox % STORE_BUFS) * STORE_BOX_BYTES);
          if (lane == 0) ptx::bulk_wait_read<STORE_BUFS - 1>();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t a = box + (uint32_t)(lane * 128 + ((q ^ (lane & 7)) << 4));
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[4 * q]),
                         "f"(v[4 * q + 1]), "f"(v[4 * q + 2]), "f"(v[4 * q + 3])
                         : "memory");
          }
          ptx::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmC, (int)n, (int)(m - lane), box);
            ptx::bulk_commit();
          }
          ++nbox;
          if (m < p.M) lse_chunk(p, n, v, rmax, rsum);
        } else if (m < p.M && n < p.N) {
          epilogue32<KIND>(p, m, mo, n, v, escale);
          if (KIND == kEpiF32Lse) lse_chunk(p, n, v, rmax, rsum);
        }
      }
      // one partial per row, column tile and half: 2 n_tiles per row
      const int64_t pidx = ((int64_t)m * p.n_tiles + n_blk) * 2 + half;
      if (KIND == kEpiF32Lse && m < p.M) p.e.lsep[pidx] = make_float2(rmax, rsum);
      if (KIND == kEpiReward && m < p.M) p.e.part[pidx] = s_row;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          ptx::mbar_arrive_cluster(acc ? tempty1 : tempty0);
        else
          ptx::mbar_arrive(acc ? tempty1 : tempty0);
      }
    }
    // the boxes' stores have left shared memory and completed before the CTA
    // (and its shared memory) goes away
    if (C::STORE && lane == 0) ptx::bulk_wait<0>();
  }

  ptx::tc_fence_before();
  // neither CTA of a pair leaves while the other may still signal its barriers
  if (PAIR) ptx::cluster_sync(); else __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) {
    if (PAIR)
      ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
    else
      ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
  }
  return fn;
}

// Row-major bf16 (or fp16) matrix (rows x cols, row stride ld elements) as a
// TMA map with a box of 64 columns x box_rows rows and 128-byte swizzling.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
              int box_rows, bool f16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major fp32 matrix (rows x cols, row stride ld elements) as a TMA store
// map: 32 x 32 boxes, 128-byte swizzling.
bool make_map_f32(CUtensorMap* map, const float* ptr, int64_t rows, int64_t cols, int64_t ld) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {(cuuint32_t)STORE_BOX, (cuuint32_t)STORE_BOX};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, bool PAIR>
cudaError_t launch_kind(cudaStream_t st, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& c, const TcParams& p, int sm_count) {
  auto fn = k_gemm_tc<KIND, PAIR>;
  constexpr size_t smem = Cfg<PAIR, KIND>::SMEM;
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int tiles = p.m_tiles * p.n_tiles;
  if (!PAIR) {
    const int grid = tiles < sm_count ? tiles : sm_count;
    fn<<<grid, THREADS, smem, st>>>(a, b, c, p);
    return cudaGetLastError();
  }
  const int pairs = tiles < sm_count / 2 ? tiles : sm_count / 2;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, fn, a, b, c, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

bool tc_gemm_supported(const GemmDesc& g, const EpiDesc& e) {
  if (g.dtype != DUST_BF16 || g.b_row_mul != 0) return false;
  // MN-major or fp16 operands: the plain fp32 epilogue only
  if ((!g.a_kmajor || !g.b_kmajor || g.f16) && e.kind != kEpiF32) return false;
  if (g.M < 1 || g.N < 16 || g.K < 8) return false;
  if ((g.lda & 7) || (g.ldb & 7)) return false;
  if (((uintptr_t)g.A & 15) || ((uintptr_t)g.B & 15)) return false;
  if (g.M > (int64_t)INT32_MAX || g.N > (int64_t)INT32_MAX || g.K > (int64_t)INT32_MAX) return false;
  if (e.kind == kEpiResidSplit && !e.resid) return false;
  if (e.kind == kEpiReward && (!e.P || !e.y || !e.part || !e.dzy || e.draws < 1)) return false;
  if (e.kind == kEpiF32Lse && !e.lsep) return false;
  if (!encode_fn()) return false;
  return e.kind == kEpiF32 || e.kind == kEpiBF16 || e.kind == kEpiGeluSplit ||
         e.kind == kEpiResidSplit || e.kind == kEpiSplit || e.kind == kEpiReward ||
         e.kind == kEpiF32Lse;
}

namespace {

template <bool PAIR>
cudaError_t launch_pair(cudaStream_t st, const GemmDesc& g, const EpiDesc& e, int sm_count,
                        uint32_t* status, uint64_t wait_ns) {
  CUtensorMap ma, mb, mc;
  const bool ok_a = g.a_kmajor ? make_map(&ma, g.A, g.M, g.K, g.lda, BM, g.f16)
                               : make_map(&ma, g.A, g.K, g.M, g.lda, BK, g.f16);
  const bool ok_b = g.b_kmajor ? make_map(&mb, g.B, g.N, g.K, g.ldb, Cfg<PAIR, kEpiF32>::B_ROWS, g.f16)
                               : make_map(&mb, g.B, g.K, g.N, g.ldb, BK, g.f16);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  memset(&mc, 0, sizeof(mc));
  // kEpiF32Lse stores C through a TMA map when its rows are 16-byte aligned
  // (else the direct per-row stores run)
  const bool tma_store = e.kind == kEpiF32Lse && ((uintptr_t)e.C & 15) == 0 &&
                         (e.ldc & 3) == 0 && make_map_f32(&mc, e.C, g.M, g.N, e.ldc);
  TcParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.m_tiles = (int)((g.M + Cfg<PAIR, kEpiF32>::TILE_M - 1) / Cfg<PAIR, kEpiF32>::TILE_M);
  p.tma_store = tma_store ? 1 : 0;
  p.f16 = g.f16 ? 1 : 0;
  p.a_mn = g.a_kmajor ? 0 : 1;
  p.b_mn = g.b_kmajor ? 0 : 1;
  p.n_tiles = (int)((g.N + BN - 1) / BN);
  p.num_kb = (int)((g.K + BK - 1) / BK);
  p.e = e;
  p.status = status;
  p.wait_ns = wait_ns;
  if (!p.status) return cudaErrorInvalidValue;
  switch (e.kind) {
    case kEpiF32: return launch_kind<kEpiF32, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiBF16: return launch_kind<kEpiBF16, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiGeluSplit: return launch_kind<kEpiGeluSplit, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiResidSplit: return launch_kind<kEpiResidSplit, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiSplit: return launch_kind<kEpiSplit, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiReward: return launch_kind<kEpiReward, PAIR>(st, ma, mb, mc, p, sm_count);
    case kEpiF32Lse: return launch_kind<kEpiF32Lse, PAIR>(st, ma, mb, mc, p, sm_count);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemm_tc(cudaStream_t st, const GemmDesc& g, const EpiDesc& e, int sm_count,
                           uint32_t* status, bool pair, uint64_t wait_ns) {
  if (wait_ns == 0) wait_ns = kWaitLimitNs;
  if (wait_ns == kWaitLimitOff) wait_ns = 0;  // injected failure: one poll per pipeline wait
  if (pair && sm_count >= 2) return launch_pair<true>(st, g, e, sm_count, status, wait_ns);
  return launch_pair<false>(st, g, e, sm_count, status, wait_ns);
}

}  // namespace dust
