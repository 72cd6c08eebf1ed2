// CUDA-core GEMM C = A B^T with fp32 accumulation: the fp32 path of the
// estimator (clean logits and G_W for fp32 inputs) and the general fallback
// for shapes the tensor-core kernel does not take.
#include "internal.cuh"

namespace dust {
namespace {

constexpr int BM = 128, BN = 128, BKT = 16, PAD = 4;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }

// Loads the A (or B) tile of rows [r0, r0+128) and k in [k0, k0+16) into
// S[k][row] as fp32, zero-filling outside the matrix.
template <typename TI, bool KMAJOR>
__device__ __forceinline__ void load_tile(float (*S)[BM + PAD], const TI* __restrict__ X,
                                          int64_t ld, int64_t rows, int64_t kdim, int64_t r0,
                                          int64_t k0, int64_t row_mul) {
  const int tid = threadIdx.x;
  if (KMAJOR) {
    const int r = tid >> 1;
    const int kk0 = (tid & 1) * 8;
    const int64_t row = r0 + r;
    int64_t src = row;
    if (row_mul != 0 && row < rows) src = (int64_t)(((unsigned long long)row * (unsigned long long)row_mul) % (unsigned long long)rows);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int64_t k = k0 + kk0 + q;
      float v = 0.0f;
      if (row < rows && k < kdim) v = to_f(X[src * ld + k]);
      S[kk0 + q][r] = v;
    }
  } else {
    const int kk = tid >> 4;
    const int rr0 = (tid & 15) * 8;
    const int64_t k = k0 + kk;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int64_t row = r0 + rr0 + q;
      float v = 0.0f;
      if (row < rows && k < kdim) v = to_f(X[k * ld + row]);
      S[kk][rr0 + q] = v;
    }
  }
}

template <typename TI, bool AK, bool BK>
__global__ __launch_bounds__(256) void k_gemm_simt(GemmDesc g, EpiDesc e) {
  __shared__ __align__(16) float As[BKT][BM + PAD];
  __shared__ __align__(16) float Bs[BKT][BN + PAD];
  const TI* A = (const TI*)g.A;
  const TI* B = (const TI*)g.B;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int64_t n0 = (int64_t)blockIdx.x * BN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  for (int64_t k0 = 0; k0 < g.K; k0 += BKT) {
    load_tile<TI, AK>(As, A, g.lda, g.M, g.K, m0, k0, 0);
    load_tile<TI, BK>(Bs, B, g.ldb, g.N, g.K, n0, k0, BK ? g.b_row_mul : 0);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BKT; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  const float escale = (e.kind == kEpiF32 && e.scale) ? *e.scale : 1.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (m >= g.M) continue;
    int64_t mo = m;
    if (e.c_row_mul != 0)
      mo = (int64_t)(((unsigned long long)m * (unsigned long long)e.c_row_mul) % (unsigned long long)g.M);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (n >= g.N) continue;
      const float v = acc[i][j];
      switch (e.kind) {
        case kEpiF32:
          e.C[mo * e.ldc + n] = v * escale;
          break;
        case kEpiBF16:
          e.Cb[m * e.ldcb + n] = __float2bfloat16_rn(v);
          break;
        case kEpiGeluSplit:
          e.C[m * e.ldc + n] = v;
          split_bf16(gelu64((double)v), &e.Cb[m * e.ldcb + n], &e.Cb[m * e.ldcb + e.split + n]);
          break;
        case kEpiResidSplit: {
          double r = (double)to_f(((const TI*)e.resid)[m * e.ldr + n]);
          if (e.rsplit > 0) r += (double)to_f(((const TI*)e.resid)[m * e.ldr + e.rsplit + n]);
          split_bf16(r + (double)v, &e.Cb[m * e.ldcb + n], &e.Cb[m * e.ldcb + e.split + n]);
          break;
        }
        case kEpiSplit:
          split_bf16(v, &e.Cb[m * e.ldcb + n], &e.Cb[m * e.ldcb + e.split + n]);
          break;
      }
    }
  }
}

template <typename TI>
cudaError_t dispatch(cudaStream_t st, const GemmDesc& g, const EpiDesc& e) {
  dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM));
  if (g.a_kmajor && g.b_kmajor) k_gemm_simt<TI, true, true><<<grid, 256, 0, st>>>(g, e);
  else if (g.a_kmajor && !g.b_kmajor) k_gemm_simt<TI, true, false><<<grid, 256, 0, st>>>(g, e);
  else if (!g.a_kmajor && g.b_kmajor) k_gemm_simt<TI, false, true><<<grid, 256, 0, st>>>(g, e);
  else k_gemm_simt<TI, false, false><<<grid, 256, 0, st>>>(g, e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_simt(cudaStream_t st, const GemmDesc& g, const EpiDesc& e) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.dtype == DUST_BF16 && g.f16) return dispatch<__half>(st, g, e);
  if (g.dtype == DUST_BF16) return dispatch<__nv_bfloat16>(st, g, e);
  return dispatch<float>(st, g, e);
}

}  // namespace dust
