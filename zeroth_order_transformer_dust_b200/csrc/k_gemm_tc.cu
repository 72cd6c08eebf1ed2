// Tensor-core GEMM for sm_100a: C = A B^T with bf16 operands and fp32
// accumulation, A (M x K) and B (N x K) both K-major.
//
// Persistent, warp-specialised CTA (one per SM): warp 0 issues TMA tile loads
// into a 4-stage shared-memory ring, warp 1 issues tcgen05.mma (128 x 256 x 16)
// into one of two TMEM accumulators, warps 2-5 drain the other accumulator
// with tcgen05.ld and run the epilogue, so the epilogue of tile i overlaps
// the MMAs of tile i+1. Every mbarrier wait is bounded in time: on expiry the
// CTA raises the timeout bit of the device status word, drains its own
// copies and MMAs (bounded again), frees its TMEM and returns.
#include <cfloat>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "tc_ptx.cuh"

namespace dust {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
static_assert(BN == kTcTileN, "reward partials are laid out per BN-column tile");
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int THREADS = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// Reward epilogue: each epilogue warp stages the probability rows of the (at
// most two) tokens its 32 rows belong to, BN columns each, per accumulator.
constexpr int PSTAGE_FLOATS = 2 * BN;
constexpr size_t PSTAGE_BYTES = (size_t)4 * 2 * PSTAGE_FLOATS * 4;  // 4 warps x 2 accumulators
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + PSTAGE_BYTES;

struct TcParams {
  int64_t M, N, K;
  int m_tiles, n_tiles, num_kb;
  EpiDesc e;
  uint32_t* status;
};

struct Shared {
  uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Shared) <= 256, "barrier block overlaps the staging area");

__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
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
                                           const float* v) {
  const EpiDesc& e = p.e;
  const bool full = n + 32 <= p.N;
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
  if (KIND == kEpiGeluSplit || KIND == kEpiResidSplit) {
    __nv_bfloat16* hi = e.Cb + m * e.ldcb + n;
    __nv_bfloat16* lo = hi + e.split;
    const __nv_bfloat16* r = KIND == kEpiResidSplit ? (const __nv_bfloat16*)e.resid + m * e.ldr + n : nullptr;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (n + q < p.N) {
        const double x = KIND == kEpiGeluSplit ? gelu64((double)v[q])
                                               : (double)__bfloat162float(r[q]) + (double)v[q];
        split_bf16(x, hi + q, lo + q);
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
        if (n + q < p.N) split_bf16((double)v[q], hi + q, lo + q);
    }
  }
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

// expm1 of a perturbed logit: degree-5 Taylor polynomial below 1/16
// (relative truncation < 2e-9), the library function otherwise.
__device__ __forceinline__ float expm1_guarded(float x) {
  if (fabsf(x) < 0.0625f) {
    float q = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
    q = fmaf(x, q, 1.0f / 6.0f);
    q = fmaf(x, q, 0.5f);
    q = fmaf(x, q, 1.0f);
    return x * q;
  }
  return expm1f(x);
}

// Reward epilogue of 32 columns of row m (target column yt): returns
// sum_n P[t, n] expm1(dz_n) and records dz at the target column. prow points
// at P[t, n]: a staged shared-memory copy (zero past column N) when `staged`,
// else the row in global memory.
__device__ __forceinline__ float reward32(const TcParams& p, int64_t m, int32_t yt, int64_t n,
                                          const float* prow, bool staged, const float* v) {
  float s = 0.0f;
  if (staged || (n + 32 <= p.N && (p.N & 3) == 0)) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 pv = staged ? reinterpret_cast<const float4*>(prow)[q]
                               : __ldg(reinterpret_cast<const float4*>(prow) + q);
      s = fmaf(pv.x, expm1_guarded(v[4 * q + 0]), s);
      s = fmaf(pv.y, expm1_guarded(v[4 * q + 1]), s);
      s = fmaf(pv.z, expm1_guarded(v[4 * q + 2]), s);
      s = fmaf(pv.w, expm1_guarded(v[4 * q + 3]), s);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (n + q < p.N) s = fmaf(prow[q], expm1_guarded(v[q]), s);
  }
  if (yt >= n && yt < n + 32) {
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (n + q == yt) p.e.dzy[m] = v[q];
  }
  return s;
}

template <int KIND>
__global__ __launch_bounds__(THREADS, 1) void k_gemm_tc(const __grid_constant__ CUtensorMap tmA,
                                                        const __grid_constant__ CUtensorMap tmB,
                                                        TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* basep = smem_raw + (base - raw);
  const uint32_t sA = base;                           // STAGES x A tile
  const uint32_t sB = base + STAGES * A_BYTES;        // STAGES x B tile
  Shared* sh = reinterpret_cast<Shared*>(basep + STAGES * STAGE_BYTES);
  float* pstage = reinterpret_cast<float*>(basep + STAGES * STAGE_BYTES + 256);
  volatile int* abort = &sh->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(ptx::smem_u32(&sh->full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&sh->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(ptx::smem_u32(&sh->tfull[a]), 1);
      ptx::mbar_init(ptx::smem_u32(&sh->tempty[a]), 4);
    }
    ptx::mbar_init(ptx::smem_u32(&sh->drain), 1);
    sh->abort = 0;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
    ptx::prefetch_map(&tmA);
    ptx::prefetch_map(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&sh->tmem_base), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // bit s: stage s holds a copy / its parity
      for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(tile, p.m_tiles, p.n_tiles, &m_blk, &n_blk);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&sh->empty[stage]), phase ^ 1u, abort, p.status)) break;
          const uint32_t fb = ptx::smem_u32(&sh->full[stage]);
          ptx::mbar_expect_tx(fb, STAGE_BYTES);
          ptx::tma_load_2d(sA + stage * A_BYTES, &tmA, kb * BK, m_blk * BM, fb);
          ptx::tma_load_2d(sB + stage * B_BYTES, &tmB, kb * BK, n_blk * BN, fb);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy this thread issued has landed before the CTA can exit
      int dummy = 0;
      for (int s = 0; s < STAGES; ++s)
        if ((armed >> s) & 1u)
          wait_bounded(ptx::smem_u32(&sh->full[s]), (armed_parity >> s) & 1u, &dummy, p.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool issued = false;
      for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&sh->tempty[acc]), acc_phase ^ 1u, abort, p.status)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&sh->full[stage]), phase, abort, p.status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sA + stage * A_BYTES, b0 = sB + stage * B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            ptx::mma_f16(d_tmem, ptx::sdesc_kmajor_sw128(a0 + k * 32),
                         ptx::sdesc_kmajor_sw128(b0 + k * 32), idesc, (kb | k) != 0);
          }
          issued = true;
          ptx::mma_commit(ptx::smem_u32(&sh->empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_u32(&sh->tfull[acc]));
      }
      if (issued) {
        // all MMAs of this CTA complete before TMEM is released
        ptx::mma_commit(ptx::smem_u32(&sh->drain));
        int dummy = 0;
        wait_bounded(ptx::smem_u32(&sh->drain), 0, &dummy, p.status);
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 ----------------
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
    const int row = quad * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
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
        const int64_t m_first = (int64_t)m_blk * BM + quad * 32;
        if (m_first < p.M && (p.N & 3) == 0) {
          const int64_t m_last = min(m_first + 31, p.M - 1);
          t_first = p.e.t0 + m_first / p.e.draws;
          const int64_t t_last = p.e.t0 + m_last / p.e.draws;
          staged = t_last - t_first <= 1;
          if (staged) {
            float4 pv[PSTAGE_FLOATS / 128];
#pragma unroll
            for (int j = 0; j < PSTAGE_FLOATS / 128; ++j) {
              const int q = lane + 32 * j;  // float4 index: token q / (BN/4), column 4 (q % (BN/4))
              const int64_t t = t_first + q / (BN / 4);
              const int64_t n = (int64_t)n_blk * BN + 4 * (q % (BN / 4));
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
      if (!wait_bounded(ptx::smem_u32(&sh->tfull[acc]), acc_phase, abort, p.status)) break;
      ptx::tc_fence_after();
      const int64_t m = (int64_t)m_blk * BM + row;
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
      for (int c = 0; c < BN / 32; ++c) {
        const int64_t n = (int64_t)n_blk * BN + c * 32;
        float v[32];
        ptx::tmem_ld32(taddr + (uint32_t)(c * 32), v);
        if (KIND == kEpiReward) {
          if (m < p.M && n < p.N) {
            const float* prow = staged ? stg + (t_row - t_first) * BN + c * 32
                                       : p.e.P + t_row * p.N + n;
            s_row += reward32(p, m, yt, n, prow, staged, v);
          }
        } else if (m < p.M && n < p.N) {
          epilogue32<KIND>(p, m, mo, n, v);
          if (KIND == kEpiF32Lse) {
            float cm = -FLT_MAX;
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (n + q < p.N) cm = fmaxf(cm, v[q]);
            const float nm = fmaxf(rmax, cm);
            float cs = 0.0f;
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (n + q < p.N) cs += __expf(v[q] - nm);
            rsum = fmaf(rsum, __expf(rmax - nm), cs);
            rmax = nm;
          }
        }
      }
      if (KIND == kEpiF32Lse && m < p.M) p.e.lsep[m * p.n_tiles + n_blk] = make_float2(rmax, rsum);
      if (KIND == kEpiReward && m < p.M) p.e.part[m * p.n_tiles + n_blk] = s_row;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&sh->tempty[acc]));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, TMEM_COLS);
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

// Row-major bf16 matrix (rows x cols, row stride ld elements) as a TMA map with
// a box of 64 columns x box_rows rows and 128-byte swizzling.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
              int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND>
cudaError_t launch_kind(cudaStream_t st, const CUtensorMap& a, const CUtensorMap& b,
                        const TcParams& p, int sm_count) {
  auto fn = k_gemm_tc<KIND>;
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
  if (err != cudaSuccess) return err;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = tiles < sm_count ? tiles : sm_count;
  fn<<<grid, THREADS, SMEM_BYTES, st>>>(a, b, p);
  return cudaGetLastError();
}

}  // namespace

bool tc_gemm_supported(const GemmDesc& g, const EpiDesc& e) {
  if (g.dtype != DUST_BF16 || !g.a_kmajor || !g.b_kmajor || g.b_row_mul != 0) return false;
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

cudaError_t launch_gemm_tc(cudaStream_t st, const GemmDesc& g, const EpiDesc& e, int sm_count,
                           uint32_t* status) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, g.A, g.M, g.K, g.lda, BM) || !make_map(&mb, g.B, g.N, g.K, g.ldb, BN))
    return cudaErrorInvalidValue;
  TcParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.m_tiles = (int)((g.M + BM - 1) / BM);
  p.n_tiles = (int)((g.N + BN - 1) / BN);
  p.num_kb = (int)((g.K + BK - 1) / BK);
  p.e = e;
  p.status = status;
  if (!p.status) return cudaErrorInvalidValue;
  switch (e.kind) {
    case kEpiF32: return launch_kind<kEpiF32>(st, ma, mb, p, sm_count);
    case kEpiBF16: return launch_kind<kEpiBF16>(st, ma, mb, p, sm_count);
    case kEpiGeluSplit: return launch_kind<kEpiGeluSplit>(st, ma, mb, p, sm_count);
    case kEpiResidSplit: return launch_kind<kEpiResidSplit>(st, ma, mb, p, sm_count);
    case kEpiSplit: return launch_kind<kEpiSplit>(st, ma, mb, p, sm_count);
    case kEpiReward: return launch_kind<kEpiReward>(st, ma, mb, p, sm_count);
    case kEpiF32Lse: return launch_kind<kEpiF32Lse>(st, ma, mb, p, sm_count);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dust
