// Full-vocabulary LM-head draws ("Dust：无需反向传播的Transformer零阶预训练",
// §1): every logit of token t gets sigma*eps; the perturbed loss is formed in
// delta form from the cached softmax p,
//   L' - L = log1p(sum_j p_j expm1(sigma eps_j)) - sigma eps_y,
// the reward is r = L - L', and g_t = -(1/(K sigma)) sum_i r_i eps_i.
// The reward needs the whole row before any g entry can be formed, so the
// noise is generated twice (stage 1 and stage 3); it never reaches memory.
#include "internal.cuh"
#include "noise.cuh"

namespace dust {
namespace {

constexpr int kWarps = 8;
constexpr int kBlocksPerWarp = 4;                     // 128-slot blocks per warp
constexpr int kSlab = kWarps * kBlocksPerWarp * 128;  // vocabulary entries per CTA
constexpr int kDrawChunk = 64;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int DEG>
__global__ __launch_bounds__(kWarps * 32) void k_full_reward_partial(
    Key key, uint32_t t_off, uint32_t i_off, uint32_t ctr3, float sigma, int64_t V, int32_t K,
    int nslab, const float* __restrict__ P, float* __restrict__ part) {
  __shared__ float sh[kWarps][kDrawChunk];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x;
  const int slab = blockIdx.y;
  const int64_t blk0 = (int64_t)slab * (kSlab / 128) + warp * kBlocksPerWarp;
  float pv[kBlocksPerWarp][4];
#pragma unroll
  for (int b = 0; b < kBlocksPerWarp; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
      pv[b][j] = pos < V ? P[t * V + pos] : 0.0f;
    }
  const uint32_t t_abs = t_off + (uint32_t)t;
  for (int i0 = 0; i0 < K; i0 += kDrawChunk) {
    const int n = min(kDrawChunk, K - i0);
    for (int ii = 0; ii < n; ++ii) {
      const uint32_t i_abs = i_off + (uint32_t)(i0 + ii);
      float s = 0.0f;
#pragma unroll
      for (int b = 0; b < kBlocksPerWarp; ++b) {
        if ((blk0 + b) * 128 < V) {
          U4 c{slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), t_abs, i_abs, ctr3};
          const G4 g = gauss4(philox10(c, key.k0, key.k1));
#pragma unroll
          for (int j = 0; j < 4; ++j) s = fmaf(pv[b][j], expm1_small<DEG>(sigma * g.v[j]), s);
        }
      }
      s = warp_sum(s);
      if (lane == 0) sh[warp][ii] = s;
    }
    __syncthreads();
    if ((int)threadIdx.x < n) {
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += sh[w][threadIdx.x];
      part[(t * nslab + slab) * (int64_t)K + i0 + threadIdx.x] = s;
    }
    __syncthreads();
  }
}

__global__ void k_full_reward_combine(Key key, uint32_t t_off, uint32_t i_off, uint32_t ctr3,
                                      float sigma, int64_t T, int64_t V, int32_t K, int nslab,
                                      const float* __restrict__ part,
                                      const int32_t* __restrict__ y, float* __restrict__ r) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= T * K) return;
  const int64_t t = id / K;
  const int32_t i = (int32_t)(id % K);
  float s = 0.0f;
  for (int sl = 0; sl < nslab; ++sl) s += part[(t * nslab + sl) * (int64_t)K + i];
  int32_t yt = y[t];
  if (yt < 0 || (int64_t)yt >= V) yt = 0;  // reported by the loss kernel
  const float ey = gauss_slot(key, t_off + (uint32_t)t, i_off + (uint32_t)i, ctr3, (uint32_t)yt);
  r[id] = sigma * ey - log1pf(s);
}

template <typename TO>
__global__ __launch_bounds__(kWarps * 32) void k_full_g(Key key, uint32_t t_off, uint32_t i_off,
                                                        uint32_t ctr3, float scale, int64_t V,
                                                        int32_t K, const float* __restrict__ r,
                                                        float* __restrict__ g_out,
                                                        TO* __restrict__ gop, int64_t plane) {
  __shared__ float rs[1024];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x;
  const int64_t blk0 = (int64_t)blockIdx.y * (kSlab / 128) + warp * kBlocksPerWarp;
  const uint32_t t_abs = t_off + (uint32_t)t;
  float acc[kBlocksPerWarp][4];
#pragma unroll
  for (int b = 0; b < kBlocksPerWarp; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[b][j] = 0.0f;
  for (int i0 = 0; i0 < K; i0 += 1024) {
    const int n = min(1024, K - i0);
    __syncthreads();
    for (int q = threadIdx.x; q < n; q += blockDim.x) rs[q] = r[t * K + i0 + q];
    __syncthreads();
    for (int ii = 0; ii < n; ++ii) {
      const float ri = rs[ii];
      const uint32_t i_abs = i_off + (uint32_t)(i0 + ii);
#pragma unroll
      for (int b = 0; b < kBlocksPerWarp; ++b) {
        if ((blk0 + b) * 128 < V) {
          U4 c{slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), t_abs, i_abs, ctr3};
          const G4 g = gauss4(philox10(c, key.k0, key.k1));
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[b][j] = fmaf(ri, g.v[j], acc[b][j]);
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kBlocksPerWarp; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
      if (pos < V) {
        const float v = acc[b][j] * scale;
        if (g_out) g_out[t * V + pos] = v;
        store_g_operand(gop, plane, t * V + pos, v);
      }
    }
}

int expm1_degree(float sigma) {
  const float xmax = sigma * 5.7686f;  // |eps| <= sqrt(48 ln 2)
  if (xmax <= 0.03f) return 4;
  if (xmax <= 0.06f) return 5;
  return 0;
}

}  // namespace

int full_vocab_nslab(int64_t V) { return (int)((V + kSlab - 1) / kSlab); }

cudaError_t launch_full_reward_partial(cudaStream_t st, const dust_params& p, const float* P,
                                       float* part) {
  const int nslab = full_vocab_nslab(p.V);
  dim3 grid((unsigned)p.T, (unsigned)nslab);
  const Key key = key_of(p.seed);
  const uint32_t c3 = ctr3_of(kTagHead, p.stream_id);
  switch (expm1_degree(p.sigma)) {
    case 4:
      k_full_reward_partial<4><<<grid, kWarps * 32, 0, st>>>(key, (uint32_t)p.token_offset,
          (uint32_t)p.draw_offset, c3, p.sigma, p.V, p.K, nslab, P, part);
      break;
    case 5:
      k_full_reward_partial<5><<<grid, kWarps * 32, 0, st>>>(key, (uint32_t)p.token_offset,
          (uint32_t)p.draw_offset, c3, p.sigma, p.V, p.K, nslab, P, part);
      break;
    default:
      k_full_reward_partial<0><<<grid, kWarps * 32, 0, st>>>(key, (uint32_t)p.token_offset,
          (uint32_t)p.draw_offset, c3, p.sigma, p.V, p.K, nslab, P, part);
  }
  return cudaGetLastError();
}

cudaError_t launch_full_reward_combine(cudaStream_t st, const dust_params& p, const float* part,
                                       const int32_t* y, float* r) {
  const int64_t n = p.T * (int64_t)p.K;
  const int threads = 256;
  k_full_reward_combine<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
      key_of(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
      ctr3_of(kTagHead, p.stream_id), p.sigma, p.T, p.V, p.K, full_vocab_nslab(p.V), part, y, r);
  return cudaGetLastError();
}

cudaError_t launch_full_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                          void* gop) {
  dim3 grid((unsigned)p.T, (unsigned)full_vocab_nslab(p.V));
  const float scale = p.sigma > 0.0f ? -1.0f / ((float)p.K * p.sigma) : 0.0f;
  const Key key = key_of(p.seed);
  const uint32_t c3 = ctr3_of(kTagHead, p.stream_id);
  const int64_t plane = p.T * p.V;
  if (p.dtype == DUST_BF16)
    k_full_g<__nv_bfloat16><<<grid, kWarps * 32, 0, st>>>(key, (uint32_t)p.token_offset,
        (uint32_t)p.draw_offset, c3, scale, p.V, p.K, r, g_out, (__nv_bfloat16*)gop, plane);
  else
    k_full_g<float><<<grid, kWarps * 32, 0, st>>>(key, (uint32_t)p.token_offset,
        (uint32_t)p.draw_offset, c3, scale, p.V, p.K, r, g_out, (float*)gop, plane);
  return cudaGetLastError();
}

}  // namespace dust
