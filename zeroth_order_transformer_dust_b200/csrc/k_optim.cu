// SGD with momentum on the weights the estimator produced a gradient for.
//
// The Dust pages train under SGD with momentum ("Dust：无需反向传播的Transformer
// 零阶预训练", §2 实证发现) without stating its form; this is the heavy-ball
// step with no dampening, Nesterov term or weight decay:
//   v <- mu v + G,   W <- W - lr v
// on fp32 master weights, optionally refreshing a bf16 copy (round to nearest
// even) that the next estimator call reads. Purely streaming: 12 bytes read
// and 8 (+2 with the copy) written per element, so the kernel is HBM-bound;
// grid-stride over float4 groups, sized to fill every SM.
#include "internal.cuh"

namespace dust {
namespace {

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, float4 w) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(w.x, w.y);
  const __nv_bfloat162 b = __floats2bfloat162_rn(w.z, w.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

__global__ __launch_bounds__(256) void k_sgd_momentum(int64_t n, float lr, float mu,
                                                      const float* __restrict__ G,
                                                      float* __restrict__ v,
                                                      float* __restrict__ W,
                                                      __nv_bfloat16* __restrict__ Wb) {
  const int64_t n4 = n >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 g = __ldcs(reinterpret_cast<const float4*>(G) + i);
    float4 m = __ldcs(reinterpret_cast<const float4*>(v) + i);
    float4 w = __ldcs(reinterpret_cast<const float4*>(W) + i);
    m.x = fmaf(mu, m.x, g.x);
    m.y = fmaf(mu, m.y, g.y);
    m.z = fmaf(mu, m.z, g.z);
    m.w = fmaf(mu, m.w, g.w);
    w.x = fmaf(-lr, m.x, w.x);
    w.y = fmaf(-lr, m.y, w.y);
    w.z = fmaf(-lr, m.z, w.z);
    w.w = fmaf(-lr, m.w, w.w);
    __stcs(reinterpret_cast<float4*>(v) + i, m);
    __stcs(reinterpret_cast<float4*>(W) + i, w);
    if (Wb) store_bf16x4(Wb + 4 * i, w);
  }
  // ragged tail (n not a multiple of 4)
  const int64_t i = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float m = fmaf(mu, v[i], G[i]);
    const float w = fmaf(-lr, m, W[i]);
    v[i] = m;
    W[i] = w;
    if (Wb) Wb[i] = __float2bfloat16_rn(w);
  }
}

}  // namespace

cudaError_t launch_sgd_momentum(cudaStream_t st, int64_t n, float lr, float mu, const float* G,
                                float* v, float* W, __nv_bfloat16* Wb, int sm_count) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t groups = (n + 3) / 4;
  int64_t blocks = (groups + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count * 8;  // 8 CTAs of 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  k_sgd_momentum<<<(unsigned)blocks, threads, 0, st>>>(n, lr, mu, G, v, W, Wb);
  return cudaGetLastError();
}

}  // namespace dust
