// Layout kernels feeding the tensor-core GEMMs: a 2-byte transpose (the
// token-major g and H become K-major operands of G_W = g^T H where their rows
// cannot be read MN-major), a row gather that permutes the head weight for
// subset draws (row q of the copy is row (a q) mod V of W, so the clean
// logits come out in permuted column order), and the conversion of H to
// fp16 with a power-of-two scale for the G_W GEMM on the fp16 g operand.
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

// Largest |x| over n bf16 values into *absmax as float bits (non-negative
// floats order like their bits, so an integer atomicMax orders them):
// 8 values per 16-byte load, a warp maximum, one atomic per warp.
__global__ __launch_bounds__(256) void k_absmax_bf16(const __nv_bfloat16* __restrict__ x,
                                                     int64_t n, uint32_t* absmax) {
  float m = 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t done = 0;
  if ((reinterpret_cast<uintptr_t>(x) & 15) == 0) {
    const int64_t n8 = n / 8;
    const uint4* x8 = reinterpret_cast<const uint4*>(x);
    for (int64_t i = i0; i < n8; i += stride) {
      const uint4 u = x8[i];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[h]);
        m = fmaxf(m, fmaxf(fabsf(__low2float(b)), fabsf(__high2float(b))));
      }
    }
    done = n8 * 8;
  }
  for (int64_t i = done + i0; i < n; i += stride) m = fmaxf(m, fabsf(__bfloat162float(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(absmax, __float_as_uint(m));
}

// The shift s that puts the largest magnitude m in [2^14, 2^15) (0 for a zero
// or non-finite m), clamped so that 2^-s and 2^s stay normal floats.
__device__ __forceinline__ int f16_shift(uint32_t bits) {
  const float m = __uint_as_float(bits);
  if (!(m > 0.0f) || isinf(m)) return 0;
  int e;
  frexpf(m, &e);  // m = f 2^e, f in [1/2, 1): floor(log2 m) = e - 1
  return max(-100, min(113, e - 1 - 14));
}

// dst = fp16(x 2^-s): exact for every x whose scaled magnitude is at least
// 2^-14 (bf16 carries 8 significant bits, fp16 11), subnormal below.
__global__ __launch_bounds__(256) void k_to_f16_scaled(const __nv_bfloat16* __restrict__ x,
                                                       int64_t n, const uint32_t* absmax,
                                                       float g_scale, __half* __restrict__ dst,
                                                       float* epi_scale) {
  const int s = f16_shift(*absmax);
  const float f = ldexpf(1.0f, -s);
  if (blockIdx.x == 0 && threadIdx.x == 0) *epi_scale = ldexpf(1.0f, s) / g_scale;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t done = 0;
  if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0) {
    const int64_t n8 = n / 8;
    const uint4* x8 = reinterpret_cast<const uint4*>(x);
    uint4* d8 = reinterpret_cast<uint4*>(dst);
    for (int64_t i = i0; i < n8; i += stride) {
      const uint4 u = x8[i];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[h]);
        const __half2 c = __floats2half2_rn(__low2float(b) * f, __high2float(b) * f);
        o[h] = *reinterpret_cast<const uint32_t*>(&c);
      }
      d8[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    done = n8 * 8;
  }
  for (int64_t i = done + i0; i < n; i += stride) dst[i] = __float2half_rn(__bfloat162float(x[i]) * f);
}

unsigned grid_for(int64_t n) {
  const int64_t blocks = (n / 8 + 255) / 256;
  return (unsigned)(blocks < 1 ? 1 : (blocks > 2368 ? 2368 : blocks));
}

}  // namespace

cudaError_t launch_absmax_bf16(cudaStream_t st, const __nv_bfloat16* x, int64_t n,
                               uint32_t* absmax) {
  if (n <= 0) return cudaSuccess;
  k_absmax_bf16<<<grid_for(n), 256, 0, st>>>(x, n, absmax);
  return cudaGetLastError();
}

cudaError_t launch_to_f16_scaled(cudaStream_t st, const __nv_bfloat16* x, int64_t n,
                                 const uint32_t* absmax, float g_scale, __half* dst,
                                 float* epi_scale) {
  k_to_f16_scaled<<<grid_for(n), 256, 0, st>>>(x, n, absmax, g_scale, dst, epi_scale);
  return cudaGetLastError();
}

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
