// Debug kernels exposing the raw Philox stream and the Gaussian slots.
#include "internal.cuh"
#include "noise.cuh"

namespace dust {

__global__ void k_debug_philox(uint64_t seed, const uint32_t* __restrict__ ctr, int64_t n,
                               uint32_t* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const Key key = key_of(seed);
  U4 c{ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3]};
  const U4 w = philox10(c, key.k0, key.k1);
  out[4 * i] = w.x;
  out[4 * i + 1] = w.y;
  out[4 * i + 2] = w.z;
  out[4 * i + 3] = w.w;
}

cudaError_t launch_debug_philox(cudaStream_t st, uint64_t seed, const uint32_t* ctr, int64_t n,
                                uint32_t* out) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  k_debug_philox<<<(unsigned)blocks, threads, 0, st>>>(seed, ctr, n, out);
  return cudaGetLastError();
}

// One thread per (token, draw, counter block of 128 slots, lane): one Philox
// call gives slots lane, lane+32, lane+64, lane+96 of the block.
__global__ void k_debug_gauss(Key key, uint32_t t_off, uint32_t i_off, uint32_t ctr3, int64_t nt,
                              int64_t ni, int64_t nslots, float* __restrict__ out) {
  const int64_t nblk = (nslots + 127) / 128;
  const int64_t total = nt * ni * nblk * 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= total) return;
  const uint32_t lane = (uint32_t)(gid & 31);
  int64_t rest = gid >> 5;
  const int64_t blk = rest % nblk;
  rest /= nblk;
  const int64_t i = rest % ni;
  const int64_t t = rest / ni;
  U4 c{slot_ctr0((uint32_t)blk, lane), t_off + (uint32_t)t, i_off + (uint32_t)i, ctr3};
  const G4 g = gauss4(philox10(c, key.k0, key.k1));
  float* row = out + (t * ni + i) * nslots;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t k = blk * 128 + lane + 32 * j;
    if (k < nslots) row[k] = g.v[j];
  }
}

// Same with the table-driven angle step of the draw kernels (packed: the
// fp32x2 form they use; else the scalar form); grid-stride so that each CTA
// builds its table once.
__global__ __launch_bounds__(256) void k_debug_gauss_tab(Key key, uint32_t t_off, uint32_t i_off,
                                                         uint32_t ctr3, int64_t nt, int64_t ni,
                                                         int64_t nslots, float* __restrict__ out,
                                                         int packed) {
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, 1.0f);
  __syncthreads();
  const int64_t nblk = (nslots + 127) / 128;
  const int64_t total = nt * ni * nblk * 32;
  for (int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t lane = (uint32_t)(gid & 31);
    int64_t rest = gid >> 5;
    const int64_t blk = rest % nblk;
    rest /= nblk;
    const int64_t i = rest % ni;
    const int64_t t = rest / ni;
    U4 c{slot_ctr0((uint32_t)blk, lane), t_off + (uint32_t)t, i_off + (uint32_t)i, ctr3};
    const U4 w = philox10(c, key.k0, key.k1);
    G4 g;
    if (packed) {
      float2 e02, e13;
      gauss4_tab_x2(w, tab, e02, e13);
      g.v[0] = e02.x;
      g.v[1] = e13.x;
      g.v[2] = e02.y;
      g.v[3] = e13.y;
    } else {
      g = gauss4_tab(w, tab);
    }
    float* row = out + (t * ni + i) * nslots;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t k = blk * 128 + lane + 32 * j;
      if (k < nslots) row[k] = g.v[j];
    }
  }
}

// Every value of the two Box-Muller inputs: radius(j) for u1 = (j + 1) 2^-24
// and (cos, sin) of 2 pi m 2^-24, with the device functions the kernels use.
// method 0: the radius sigma R as the polynomial-angle step forms it;
// method 1: rho = R / sqrt(2 ln 2), the factor the table step uses.
__global__ void k_debug_bm_radius(int method, float sigma, float* __restrict__ out) {
  const uint32_t j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < (1u << 24)) out[j] = method == 1 ? bm_rho(j << 8) : (sigma * kRhoToR) * bm_rho(j << 8);
}

__global__ __launch_bounds__(256) void k_debug_bm_angle(int method, float* __restrict__ out) {
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, 1.0f);
  __syncthreads();
  for (uint32_t m = blockIdx.x * blockDim.x + threadIdx.x; m < (1u << 24);
       m += gridDim.x * blockDim.x) {
    float s, c;
    if (method == 1) {
      const float2 cs = rotate_tab(m << 8, tab);
      c = cs.x;
      s = cs.y;
    } else {
      sincos_turn24(m, &s, &c);
    }
    out[2 * (size_t)m] = c;
    out[2 * (size_t)m + 1] = s;
  }
}

cudaError_t launch_debug_bm(cudaStream_t st, int what, float sigma, float* out) {
  if (what == 0 || what == 3)
    k_debug_bm_radius<<<(1u << 24) / 256, 256, 0, st>>>(what == 3 ? 1 : 0, sigma, out);
  else
    k_debug_bm_angle<<<4096, 256, 0, st>>>(what == 2 ? 1 : 0, out);
  return cudaGetLastError();
}

cudaError_t launch_debug_gauss(cudaStream_t st, const dust_params& p, int tag, int64_t nt,
                               int64_t ni, int64_t nslots, float* out, int method) {
  const int64_t nblk = (nslots + 127) / 128;
  const int64_t total = nt * ni * nblk * 32;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (method == 1 || method == 2) {
    k_debug_gauss_tab<<<(unsigned)(blocks < 2048 ? blocks : 2048), threads, 0, st>>>(
        key_of(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
        ctr3_of(tag, p.stream_id), nt, ni, nslots, out, method == 1);
  } else {
    k_debug_gauss<<<(unsigned)blocks, threads, 0, st>>>(
        key_of(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
        ctr3_of(tag, p.stream_id), nt, ni, nslots, out);
  }
  return cudaGetLastError();
}

}  // namespace dust
