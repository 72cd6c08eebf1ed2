// Layout kernels feeding the tensor-core GEMMs: a bf16 transpose (the
// token-major g and H become the K-major operands of G_W = g^T H) and a row
// gather that permutes the head weight for subset draws (row q of the copy is
// row (a q) mod V of W, so the clean logits come out in permuted column order).
#include "internal.cuh"

namespace dust {
namespace {

constexpr int TT = 64;

__global__ __launch_bounds__(256) void k_transpose_bf16(const __nv_bfloat16* __restrict__ src,
                                                        int64_t rows, int64_t cols,
                                                        __nv_bfloat16* __restrict__ dst,
                                                        int64_t ld_dst) {
  __shared__ __nv_bfloat16 tile[TT][TT + 2];
  const int64_t r0 = (int64_t)blockIdx.x * TT;  // source rows = destination columns
  const int64_t c0 = (int64_t)blockIdx.y * TT;  // source columns = destination rows
  for (int i = threadIdx.x; i < TT * TT; i += blockDim.x) {
    const int rr = i / TT, cc = i % TT;
    const int64_t r = r0 + rr, c = c0 + cc;
    tile[rr][cc] = (r < rows && c < cols) ? src[r * cols + c] : __float2bfloat16_rn(0.0f);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < TT * TT; i += blockDim.x) {
    const int cc = i / TT, rr = i % TT;
    const int64_t drow = c0 + cc, dcol = r0 + rr;
    if (drow < cols && dcol < ld_dst) dst[drow * ld_dst + dcol] = tile[rr][cc];
  }
}

// dst[q] = src[(q * mul) mod rows], rows of `cols` bf16 elements, 16-byte moves.
__global__ void k_permute_rows_bf16(const __nv_bfloat16* __restrict__ src, int64_t rows,
                                    int64_t cols, int64_t mul, __nv_bfloat16* __restrict__ dst) {
  const int64_t q = blockIdx.x;
  const int64_t s = (int64_t)(((unsigned long long)q * (unsigned long long)mul) %
                              (unsigned long long)rows);
  const __nv_bfloat16* a = src + s * cols;
  __nv_bfloat16* b = dst + q * cols;
  if ((cols & 7) == 0 && (((uintptr_t)src | (uintptr_t)dst) & 15) == 0) {
    const uint4* a4 = reinterpret_cast<const uint4*>(a);
    uint4* b4 = reinterpret_cast<uint4*>(b);
    for (int64_t j = threadIdx.x; j < cols / 8; j += blockDim.x) b4[j] = a4[j];
  } else {
    for (int64_t j = threadIdx.x; j < cols; j += blockDim.x) b[j] = a[j];
  }
}

}  // namespace

cudaError_t launch_transpose_bf16(cudaStream_t st, const __nv_bfloat16* src, int64_t rows,
                                  int64_t cols, __nv_bfloat16* dst, int64_t ld_dst) {
  dim3 grid((unsigned)((ld_dst + TT - 1) / TT), (unsigned)((cols + TT - 1) / TT));
  k_transpose_bf16<<<grid, 256, 0, st>>>(src, rows, cols, dst, ld_dst);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows_bf16(cudaStream_t st, const __nv_bfloat16* src, int64_t rows,
                                     int64_t cols, int64_t mul, __nv_bfloat16* dst) {
  k_permute_rows_bf16<<<(unsigned)rows, 128, 0, st>>>(src, rows, cols, mul, dst);
  return cudaGetLastError();
}

}  // namespace dust
