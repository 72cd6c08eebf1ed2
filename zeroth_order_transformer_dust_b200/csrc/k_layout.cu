// Layout kernels feeding the tensor-core GEMMs: a bf16 transpose (the
// token-major g and H become the K-major operands of G_W = g^T H) and a row
// gather that permutes the head weight for subset draws (row q of the copy is
// row (a q) mod V of W, so the clean logits come out in permuted column order).
#include "internal.cuh"

namespace dust {
namespace {

constexpr int TT = 64;

// dst[c * ld_dst + r] = src[r * cols + c] for r < ld_dst (zero for r >= rows),
// through a 64 x 64 shared-memory tile. Vector path (cols and ld_dst multiples
// of 8, 16-byte aligned bases): every thread moves 16 bytes per global load
// and per global store; the tile row pitch of 33 words keeps the 8-row column
// gathers of the store phase at most two-way bank conflicted.
__global__ __launch_bounds__(256) void k_transpose_bf16_v8(const __nv_bfloat16* __restrict__ src,
                                                           int64_t rows, int64_t cols,
                                                           __nv_bfloat16* __restrict__ dst,
                                                           int64_t ld_dst) {
  __shared__ uint32_t tile[TT][TT / 2 + 1];  // bf16 pairs
  const int64_t r0 = (int64_t)blockIdx.x * TT;  // source rows = destination columns
  const int64_t c0 = (int64_t)blockIdx.y * TT;  // source columns = destination rows
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = threadIdx.x + 256 * h;
    const int rr = i >> 3, cv = i & 7;
    const int64_t r = r0 + rr, c = c0 + 8 * cv;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows && c < cols) v = *reinterpret_cast<const uint4*>(src + r * cols + c);
    tile[rr][4 * cv + 0] = v.x;
    tile[rr][4 * cv + 1] = v.y;
    tile[rr][4 * cv + 2] = v.z;
    tile[rr][4 * cv + 3] = v.w;
  }
  __syncthreads();
  const uint16_t* t16 = reinterpret_cast<const uint16_t*>(&tile[0][0]);
  constexpr int kPitch16 = 2 * (TT / 2 + 1);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = threadIdx.x + 256 * h;
    const int dc = i >> 3, rg = i & 7;  // destination row c0 + dc, columns r0 + 8 rg ..
    const int64_t drow = c0 + dc, dcol = r0 + 8 * rg;
    if (drow >= cols || dcol >= ld_dst) continue;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t lo = t16[(8 * rg + 2 * q) * kPitch16 + dc];
      const uint32_t hi = t16[(8 * rg + 2 * q + 1) * kPitch16 + dc];
      w[q] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(dst + drow * ld_dst + dcol) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Generic element-wise path (any shape or alignment).
__global__ __launch_bounds__(256) void k_transpose_bf16(const __nv_bfloat16* __restrict__ src,
                                                        int64_t rows, int64_t cols,
                                                        __nv_bfloat16* __restrict__ dst,
                                                        int64_t ld_dst) {
  __shared__ __nv_bfloat16 tile[TT][TT + 2];
  const int64_t r0 = (int64_t)blockIdx.x * TT;
  const int64_t c0 = (int64_t)blockIdx.y * TT;
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
  const bool vec = (cols % 8) == 0 && (ld_dst % 8) == 0 && (((uintptr_t)src | (uintptr_t)dst) & 15) == 0;
  if (vec)
    k_transpose_bf16_v8<<<grid, 256, 0, st>>>(src, rows, cols, dst, ld_dst);
  else
    k_transpose_bf16<<<grid, 256, 0, st>>>(src, rows, cols, dst, ld_dst);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows_bf16(cudaStream_t st, const __nv_bfloat16* src, int64_t rows,
                                     int64_t cols, int64_t mul, __nv_bfloat16* dst) {
  k_permute_rows_bf16<<<(unsigned)rows, 128, 0, st>>>(src, rows, cols, mul, dst);
  return cudaGetLastError();
}

}  // namespace dust
