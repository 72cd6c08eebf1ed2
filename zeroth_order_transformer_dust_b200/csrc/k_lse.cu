// Clean per-token loss from cached logits: row log-sum-exp, CE against the
// target, and (optionally) the softmax p = exp(z - LSE) written in place.
// "不用反向传播训练Transformer：Dust零阶优化获突破": the head is perturbed on the
// cached logits; p is what every perturbed loss of the token reuses.
#include <cfloat>

#include "internal.cuh"

namespace dust {
namespace {

constexpr int kThreads = 512;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (kThreads / 32) ? sh[lane] : (is_max ? -FLT_MAX : 0.0f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, w) : v + w;
    }
    if (lane == 0) sh[32] = v;
  }
  __syncthreads();
  const float r = sh[32];
  __syncthreads();
  return r;
}

__global__ __launch_bounds__(kThreads) void k_lse_rows(float* __restrict__ Z, int64_t V,
                                                       const int32_t* __restrict__ y,
                                                       int64_t col_mul, float* __restrict__ lse,
                                                       float* __restrict__ loss, bool to_prob,
                                                       uint32_t* status) {
  __shared__ float sh[33];
  const int64_t t = blockIdx.x;
  float* row = Z + t * V;
  float mx = -FLT_MAX;
  for (int64_t j = threadIdx.x; j < V; j += kThreads) mx = fmaxf(mx, row[j]);
  mx = block_reduce(mx, true, sh);
  float sum = 0.0f;
  for (int64_t j = threadIdx.x; j < V; j += kThreads) sum += expf(row[j] - mx);
  sum = block_reduce(sum, false, sh);
  const float l = mx + logf(sum);
  if (threadIdx.x == 0) {
    const int32_t yt = y[t];
    float lt;
    if (yt < 0 || (int64_t)yt >= V) {
      atomicOr(status, kStatusBadTarget);
      lt = __int_as_float(0x7fc00000);
    } else {
      const int64_t col = col_mul ? (int64_t)(((unsigned long long)yt * (unsigned long long)col_mul) %
                                              (unsigned long long)V)
                                  : (int64_t)yt;
      lt = l - row[col];
    }
    lse[t] = l;
    if (loss) loss[t] = lt;
  }
  if (to_prob) {
    __syncthreads();  // the target logit is read before the row is overwritten
    for (int64_t j = threadIdx.x; j < V; j += kThreads) row[j] = expf(row[j] - l);
  }
}

// One warp per row: LSE = M + log(sum_k s_k exp(m_k - M)) over the row's
// per-tile partials (m_k, s_k), M = max_k m_k; then the clean loss against
// the target column (col_mul != 0: column (y col_mul) mod V of permuted rows).
__global__ __launch_bounds__(256) void k_lse_combine(const float2* __restrict__ lsep, int ntiles,
                                                     const float* __restrict__ Z, int64_t T,
                                                     int64_t V, const int32_t* __restrict__ y,
                                                     int64_t col_mul, float* __restrict__ lse,
                                                     float* __restrict__ loss, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float2* row = lsep + t * ntiles;
  float mx = -FLT_MAX;
  for (int k = lane; k < ntiles; k += 32) mx = fmaxf(mx, row[k].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.0f;
  for (int k = lane; k < ntiles; k += 32) sum += row[k].y * expf(row[k].x - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) {
    const float l = mx + logf(sum);
    const int32_t yt = y[t];
    float lt;
    if (yt < 0 || (int64_t)yt >= V) {
      atomicOr(status, kStatusBadTarget);
      lt = __int_as_float(0x7fc00000);
    } else {
      const int64_t col = col_mul ? (int64_t)(((unsigned long long)yt * (unsigned long long)col_mul) %
                                              (unsigned long long)V)
                                  : (int64_t)yt;
      lt = l - Z[t * V + col];
    }
    lse[t] = l;
    if (loss) loss[t] = lt;
  }
}

}  // namespace

cudaError_t launch_lse_combine(cudaStream_t st, const float2* lsep, int ntiles, const float* Z,
                               int64_t T, int64_t V, const int32_t* y, int64_t col_mul,
                               float* lse, float* loss, uint32_t* status) {
  if (T <= 0) return cudaSuccess;
  k_lse_combine<<<(unsigned)((T + 7) / 8), 256, 0, st>>>(lsep, ntiles, Z, T, V, y, col_mul, lse,
                                                         loss, status);
  return cudaGetLastError();
}

cudaError_t launch_lse_rows(cudaStream_t st, float* Z, int64_t T, int64_t V, const int32_t* y,
                            int64_t col_mul, float* lse, float* loss, bool to_prob,
                            uint32_t* status) {
  if (T <= 0) return cudaSuccess;
  k_lse_rows<<<(unsigned)T, kThreads, 0, st>>>(Z, V, y, col_mul, lse, loss, to_prob, status);
  return cudaGetLastError();
}

}  // namespace dust
