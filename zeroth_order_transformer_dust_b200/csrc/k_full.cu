// Full-vocabulary LM-head draws ("Dust：无需反向传播的Transformer零阶预训练",
// §1): every logit of token t gets sigma*eps; the perturbed loss is formed in
// delta form from the softmax p = exp(z - LSE) of the cached clean logits,
//   L' - L = log1p(sum_j p_j expm1(sigma eps_j)) - sigma eps_y,
// the reward is r = L - L', and g_t = -(1/(K sigma)) sum_i r_i eps_i.
// The reward needs the whole row before any g entry can be formed, so the
// noise is generated twice (stage 1 and stage 3); it never reaches memory.
//
// Both noise passes are persistent over (token, 3072-entry slab) units: a warp
// owns three 128-slot blocks of the slab, evaluates Philox rounds 0-1 of its
// blocks once per unit and those of each draw once per draw, and turns words
// into sigma-scaled Gaussians with the table-driven Box-Muller step (the
// table of roots of unity is built once per CTA). Stage 1 also records the
// target's noise, so stage 2 needs none of its own.
#include "internal.cuh"
#include "noise.cuh"

namespace dust {
namespace {

constexpr int kWarps = 8;
// 128-slot blocks per warp: three keeps both passes within 64 registers, so
// they run 32 warps per SM (four blocks, 72 registers in the reward pass:
// 24 warps; 2 % slower on full_bf16)
constexpr int kBlocksPerWarp = 3;
constexpr int kSlab = kWarps * kBlocksPerWarp * 128;  // vocabulary entries per unit
constexpr int kDrawChunk = 64;
// The Box-Muller step in packed fp32x2 form (PACKED) or scalar and paired up
// afterwards. Packed operations run on the FMA-heavy pipe, which the Philox
// multiplies also need: measured on B200, the reward pass (with its packed
// expm1 and sums) is faster with the packed step (15.5 against 15.9 ms on
// full_bf16), the g pass with the scalar one (12.3 against 12.5 ms).
template <bool PACKED>
__device__ __forceinline__ void noise4(U4 w, const float2* tab, float2& e02, float2& e13) {
  if (PACKED) {
    gauss4_tab_x2(w, tab, e02, e13);
  } else {
    const G4 g = gauss4_tab(w, tab);
    e02 = make_float2(g.v[0], g.v[2]);
    e13 = make_float2(g.v[1], g.v[3]);
  }
}

struct FullArgs {
  RoundKeys keys;
  uint32_t t_off, i_off, ctr3;
  float sigma;
  float fac;  // g = fac * sum_i r_i (sigma eps_i)
  int64_t T, V;
  int32_t K;
  int nslab;
  const float* Z;    // clean logits (T x V)
  const float* lse;  // T
  const int32_t* y;
  float* part;       // (t * nslab + slab) * K + i
  float* xy;         // sigma eps at the target, t * K + i
  const float* r;    // rewards, t * K + i
  float* g_out;
  void* gop;
  GopFormat gf;
  int64_t plane;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Draws [i0, i0 + n) of one unit for one warp; per draw, the warp's sum goes
// to sh[warp][ii]. ALL: all kBlocksPerWarp blocks of the warp lie below V
// (every warp but the one that straddles V), so no per-block test runs in the
// draw loop. The noise, expm1 and the reward sums run in packed fp32x2
// arithmetic on the pairs of slots (lane, lane + 64) and (lane + 32, lane + 96)
// of each block (p02, p13), one pair of chains per block. No barrier inside:
// the caller's block-wide barriers are the same for every warp.
template <int DEG, bool ALL>
__device__ __forceinline__ void reward_chunk(const FullArgs& A, const float2* tab, int64_t t,
                                             int i0, int n, int nvalid,
                                             const float2 (&p02)[kBlocksPerWarp],
                                             const float2 (&p13)[kBlocksPerWarp],
                                             const BlockConst (&bc)[kBlocksPerWarp],
                                             bool warp_has_y, bool y_here, int by, int jy,
                                             float (*sh)[kDrawChunk]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t t_abs = A.t_off + (uint32_t)t;
  for (int ii = 0; ii < n; ++ii) {
    const uint32_t i_abs = A.i_off + (uint32_t)(i0 + ii);
    const DrawConst dc = draw_const(A.keys, t_abs, i_abs);
    float sb[kBlocksPerWarp];
    float xyv = 0.0f;
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      sb[b] = 0.0f;
      if (ALL || b < nvalid) {
        float2 e02, e13;
        noise4<true>(philox_from2(bc[b], dc, A.keys), tab, e02, e13);
        float2 s2 = __fmul2_rn(p02[b], expm1_small_x2<DEG>(e02));
        s2 = __ffma2_rn(p13[b], expm1_small_x2<DEG>(e13), s2);
        sb[b] = s2.x + s2.y;
        if (warp_has_y && b == by) {
          // word jy of the counter: 0, 2 in e02 and 1, 3 in e13
          const float2 e = (jy & 1) ? e13 : e02;
          xyv = (jy & 2) ? e.y : e.x;
        }
      }
    }
    if (y_here) A.xy[t * A.K + i0 + ii] = xyv;
    float s = 0.0f;
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) s += sb[b];
    s = warp_sum(s);
    if (lane == 0) sh[warp][ii] = s;
  }
}

template <int DEG>
__global__ __launch_bounds__(kWarps * 32) void k_full_reward_partial(const __grid_constant__ FullArgs A) {
  __shared__ float sh[kWarps][kDrawChunk];
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, A.sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nunits = A.T * A.nslab;
  for (int64_t unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int64_t t = unit / A.nslab;
    const int slab = (int)(unit % A.nslab);
    const int64_t blk0 = (int64_t)slab * (kSlab / 128) + warp * kBlocksPerWarp;
    // blocks of this warp below V (warp-uniform)
    const int64_t left = (A.V - blk0 * 128 + 127) / 128;
    const int nvalid = left <= 0 ? 0 : (left >= kBlocksPerWarp ? kBlocksPerWarp : (int)left);
    // p = exp(z - LSE), formed once per unit, as the packed pairs of slots
    // (lane, lane + 64) and (lane + 32, lane + 96) of each block
    float2 p02[kBlocksPerWarp], p13[kBlocksPerWarp];
    BlockConst bc[kBlocksPerWarp];
    const float lse_t = A.lse[t];
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      bc[b] = block_const(A.keys, slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), A.ctr3);
      float pv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
        pv[j] = pos < A.V ? expf(A.Z[t * A.V + pos] - lse_t) : 0.0f;
      }
      p02[b] = make_float2(pv[0], pv[2]);
      p13[b] = make_float2(pv[1], pv[3]);
    }
    // the lane holding the target's noise, if this warp's blocks contain it
    int32_t yt = A.y[t];
    if (yt < 0 || (int64_t)yt >= A.V) yt = 0;  // reported by the loss kernel
    const int64_t yb = (int64_t)yt >> 7;
    const bool warp_has_y = yb >= blk0 && yb < blk0 + kBlocksPerWarp;  // warp-uniform
    const bool y_here = warp_has_y && lane == (yt & 31);
    const int by = (int)(yb - blk0), jy = (yt >> 5) & 3;
    for (int i0 = 0; i0 < A.K; i0 += kDrawChunk) {
      const int n = min(kDrawChunk, A.K - i0);
      if (nvalid == kBlocksPerWarp)
        reward_chunk<DEG, true>(A, tab, t, i0, n, nvalid, p02, p13, bc, warp_has_y, y_here, by, jy, sh);
      else
        reward_chunk<DEG, false>(A, tab, t, i0, n, nvalid, p02, p13, bc, warp_has_y, y_here, by, jy, sh);
      __syncthreads();
      if ((int)threadIdx.x < n) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += sh[w][threadIdx.x];
        A.part[(t * A.nslab + slab) * (int64_t)A.K + i0 + threadIdx.x] = s;
      }
      __syncthreads();
    }
  }
}

__global__ void k_full_reward_combine(int64_t T, int32_t K, int nslab,
                                      const float* __restrict__ part,
                                      const float* __restrict__ xy, float* __restrict__ r) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= T * K) return;
  const int64_t t = id / K;
  const int32_t i = (int32_t)(id % K);
  float s = 0.0f;
  for (int sl = 0; sl < nslab; ++sl) s += part[(t * nslab + sl) * (int64_t)K + i];
  r[id] = xy[id] - log1pf(s);
}

// Draws [i0, i0 + n) of sum_i r_i (sigma eps_i) for one warp's blocks, with
// r staged in rs (ALL: every block lies below V), accumulated in packed pairs
// (slots lane, lane + 64 in acc02; lane + 32, lane + 96 in acc13). No barrier
// inside.
template <bool ALL>
__device__ __forceinline__ void g_chunk(const FullArgs& A, const float2* tab, int64_t t, int i0,
                                        int n, int nvalid, const BlockConst (&bc)[kBlocksPerWarp],
                                        const float* rs, float2 (&acc02)[kBlocksPerWarp],
                                        float2 (&acc13)[kBlocksPerWarp]) {
  const uint32_t t_abs = A.t_off + (uint32_t)t;
  for (int ii = 0; ii < n; ++ii) {
    const float ri = rs[ii];
    const float2 r2 = make_float2(ri, ri);
    const DrawConst dc = draw_const(A.keys, t_abs, A.i_off + (uint32_t)(i0 + ii));
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      if (ALL || b < nvalid) {
        float2 e02, e13;
        noise4<false>(philox_from2(bc[b], dc, A.keys), tab, e02, e13);
        acc02[b] = __ffma2_rn(r2, e02, acc02[b]);
        acc13[b] = __ffma2_rn(r2, e13, acc13[b]);
      }
    }
  }
}

__global__ __launch_bounds__(kWarps * 32) void k_full_g(const __grid_constant__ FullArgs A) {
  __shared__ float rs[1024];
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, A.sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nunits = A.T * A.nslab;
  for (int64_t unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int64_t t = unit / A.nslab;
    const int slab = (int)(unit % A.nslab);
    const int64_t blk0 = (int64_t)slab * (kSlab / 128) + warp * kBlocksPerWarp;
    const int64_t left = (A.V - blk0 * 128 + 127) / 128;
    const int nvalid = left <= 0 ? 0 : (left >= kBlocksPerWarp ? kBlocksPerWarp : (int)left);
    BlockConst bc[kBlocksPerWarp];
    float2 acc02[kBlocksPerWarp], acc13[kBlocksPerWarp];
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      bc[b] = block_const(A.keys, slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), A.ctr3);
      acc02[b] = make_float2(0.0f, 0.0f);
      acc13[b] = make_float2(0.0f, 0.0f);
    }
    for (int i0 = 0; i0 < A.K; i0 += 1024) {
      const int n = min(1024, A.K - i0);
      __syncthreads();
      for (int q = threadIdx.x; q < n; q += blockDim.x) rs[q] = A.r[t * A.K + i0 + q];
      __syncthreads();
      if (nvalid == kBlocksPerWarp)
        g_chunk<true>(A, tab, t, i0, n, nvalid, bc, rs, acc02, acc13);
      else
        g_chunk<false>(A, tab, t, i0, n, nvalid, bc, rs, acc02, acc13);
    }
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
        if (pos < A.V) {
          const float2 a = (j & 1) ? acc13[b] : acc02[b];
          const float v = ((j & 2) ? a.y : a.x) * A.fac;
          if (A.g_out) A.g_out[t * A.V + pos] = v;
          store_gop(A.gop, A.gf, A.plane, t * A.V + pos, v);
        }
      }
  }
}

FullArgs make_args(const dust_params& p) {
  FullArgs A{};
  A.keys = round_keys(p.seed);
  A.t_off = (uint32_t)p.token_offset;
  A.i_off = (uint32_t)p.draw_offset;
  A.ctr3 = ctr3_of(kTagHead, p.stream_id);
  A.sigma = p.sigma;
  const double s2 = (double)p.sigma * (double)p.sigma;
  A.fac = p.sigma > 0.0f ? (float)(-1.0 / ((double)p.K * s2)) : 0.0f;
  A.T = p.T;
  A.V = p.V;
  A.K = p.K;
  A.nslab = (int)((p.V + kSlab - 1) / kSlab);
  A.plane = p.T * p.V;
  return A;
}

// Persistent grid: every SM filled with as many CTAs as fit, at most one per unit.
template <typename F>
int grid_for(F kernel, int64_t units) {
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarps * 32, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cudaGetLastError();
  const int64_t g = (int64_t)sms * per_sm;
  return (int)(units < g ? units : g);
}

}  // namespace

int full_vocab_nslab(int64_t V) { return (int)((V + kSlab - 1) / kSlab); }

size_t full_vocab_xy_bytes(int64_t T, int32_t K) { return (size_t)T * K * 4; }

cudaError_t launch_full_reward_partial(cudaStream_t st, const dust_params& p, const float* Z,
                                       const float* lse, const int32_t* y, float* part,
                                       float* xy) {
  FullArgs A = make_args(p);
  A.Z = Z;
  A.lse = lse;
  A.y = y;
  A.part = part;
  A.xy = xy;
  const int64_t units = A.T * A.nslab;
  switch (expm1_degree(p.sigma)) {
    case 3:
      k_full_reward_partial<3><<<grid_for(k_full_reward_partial<3>, units), kWarps * 32, 0, st>>>(A);
      break;
    case 4:
      k_full_reward_partial<4><<<grid_for(k_full_reward_partial<4>, units), kWarps * 32, 0, st>>>(A);
      break;
    default:
      k_full_reward_partial<0><<<grid_for(k_full_reward_partial<0>, units), kWarps * 32, 0, st>>>(A);
  }
  return cudaGetLastError();
}

cudaError_t launch_full_reward_combine(cudaStream_t st, const dust_params& p, const float* part,
                                       const float* xy, float* r) {
  const int64_t n = p.T * (int64_t)p.K;
  const int threads = 256;
  k_full_reward_combine<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
      p.T, p.K, full_vocab_nslab(p.V), part, xy, r);
  return cudaGetLastError();
}

cudaError_t launch_full_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                          void* gop, GopFormat gf) {
  FullArgs A = make_args(p);
  A.r = r;
  A.g_out = g_out;
  A.gop = gop;
  A.gf = gf;
  k_full_g<<<grid_for(k_full_g, A.T * A.nslab), kWarps * 32, 0, st>>>(A);
  return cudaGetLastError();
}

}  // namespace dust
