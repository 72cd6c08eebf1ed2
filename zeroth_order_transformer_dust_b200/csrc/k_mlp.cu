// Hidden-MLP up-projection draws ("Dust：无需反向传播的Transformer零阶预训练",
// §1: noise on the linear layer's output u = W_up x; 减少干扰: only what the
// perturbation changes is recomputed from cached x, u and the clean logits):
//   da = GELU(u + sigma eps) - GELU(u)        (rows (t, i), d_ff columns)
//   dh = da W_down^T,  dz = dh W_head^T,
//   r  = dz_y - log1p(sum_j p_j expm1(dz_j)),
//   g_t = -(1/(K sigma)) sum_i r_i eps_i.
#include "internal.cuh"
#include "noise.cuh"

namespace dust {
namespace {

// GELU(u + d) - GELU(u) without cancellation. With GELU(x) = x Phi(x):
//   GELU(u + d) - GELU(u) = d Phi(u + d) + u (Phi(u + d) - Phi(u)),
// and Phi(u + d) - Phi(u) is the integral of the normal density phi over
// [u, u + d], taken by two-point Gauss-Legendre quadrature (nodes at the
// midpoint +- d / (2 sqrt 3)); its truncation is |d|^5 max|phi''''| / 4320,
// below 3e-10 for |d| <= 0.06. Larger |d| use the difference of two fp64
// GELU values.
__device__ __forceinline__ float gelu_delta(float u, float d) {
  if (fabsf(d) <= 0.0625f) {
    const float x1 = u + d;
    const float phi1 = 0.5f * erfcf(-x1 * 0.70710678118654752f);
    const float mid = fmaf(0.5f, d, u);
    const float h = d * 0.28867513459481288f;  // d / (2 sqrt 3)
    const float a = mid - h, b = mid + h;
    const float dens = expf(-0.5f * a * a) + expf(-0.5f * b * b);
    const float dphi = 0.5f * d * 0.39894228040143268f * dens;  // 1 / sqrt(2 pi)
    return fmaf(d, phi1, u * dphi);
  }
  return (float)(gelu64((double)u + (double)d) - gelu64((double)u));
}

// One thread per (row, 128-channel block, lane). The GELU difference is
// formed without cancellation (gelu_delta) and stored as bf16 hi/lo planes,
// da[row*2d_ff + c] and da[row*2d_ff + d_ff + c].
__global__ void k_mlp_delta_a(Key key, uint32_t t_off, uint32_t i_off, uint32_t ctr3, float sigma,
                              int64_t d_ff, int32_t K, const float* __restrict__ u, int64_t t0,
                              int64_t rows, __nv_bfloat16* __restrict__ da_bf,
                              float* __restrict__ da_f32) {
  const int64_t nblk = (d_ff + 127) / 128;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= rows * nblk * 32) return;
  const uint32_t lane = (uint32_t)(gid & 31);
  const int64_t rest = gid >> 5;
  const int64_t blk = rest % nblk;
  const int64_t row = rest / nblk;
  const int64_t t = t0 + row / K;
  const int32_t i = (int32_t)(row % K);
  U4 c{slot_ctr0((uint32_t)blk, lane), t_off + (uint32_t)t, i_off + (uint32_t)i, ctr3};
  const G4 g = gauss4(philox10(c, key.k0, key.k1));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t ch = blk * 128 + lane + 32 * j;
    if (ch < d_ff) {
      const float d = gelu_delta(u[t * d_ff + ch], sigma * g.v[j]);
      if (da_bf) split_bf16(d, &da_bf[row * 2 * d_ff + ch], &da_bf[row * 2 * d_ff + d_ff + ch]);
      if (da_f32) da_f32[row * d_ff + ch] = d;
    }
  }
}

// The same deltas for small perturbations (|sigma eps| <= 5.77 sigma <= 1/16):
// GELU(u + d) - GELU(u) = sum_{n=1..4} G_n(u) d^n / n! + R, where G_n is the
// n-th derivative of GELU(x) = x Phi(x):
//   G_1 = Phi + u phi,   G_2 = phi (2 - u^2),   G_3 = phi (u^3 - 4u),
//   G_4 = phi (7u^2 - u^4 - 4),
// and |R| <= max|G_5| |d|^5 / 120 < 2.3e-8 (max|G_5| = 2.84). u is the same
// for every draw of a token, so one warp takes a (token, 128-channel block),
// forms the four coefficients of its channels once in fp64, and walks the
// token's K draws with the first two Philox rounds hoisted and the
// sigma-scaled table angle step; each delta costs four FMAs.
__global__ __launch_bounds__(256) void k_mlp_delta_a_taylor(RoundKeys keys, uint32_t t_off,
                                                            uint32_t i_off, uint32_t ctr3,
                                                            float sigma, int64_t d_ff, int32_t K,
                                                            const float* __restrict__ u, int64_t t0,
                                                            int64_t nt,
                                                            __nv_bfloat16* __restrict__ da) {
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nblk = (d_ff + 127) / 128;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= nt * nblk) return;  // no block-wide barrier follows
  const int64_t tl = wid / nblk;
  const int64_t blk = wid % nblk;
  const int64_t t = t0 + tl;
  float c1[4], c2[4], c3[4], c4[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t ch = blk * 128 + lane + 32 * j;
    const double x = ch < d_ff ? (double)u[t * d_ff + ch] : 0.0;
    const double phi = 0.3989422804014327 * exp(-0.5 * x * x);
    const double Phi = 0.5 * erfc(-x * 0.7071067811865476);
    const double x2 = x * x;
    c1[j] = (float)(Phi + x * phi);
    c2[j] = (float)(phi * (2.0 - x2) * 0.5);
    c3[j] = (float)(phi * x * (x2 - 4.0) * (1.0 / 6.0));
    c4[j] = (float)(phi * (7.0 * x2 - x2 * x2 - 4.0) * (1.0 / 24.0));
  }
  const BlockConst bc = block_const(keys, slot_ctr0((uint32_t)blk, (uint32_t)lane), ctr3);
  const uint32_t t_abs = t_off + (uint32_t)t;
  for (int32_t i = 0; i < K; ++i) {
    const G4 g = gauss4_tab(philox_from2(bc, draw_const(keys, t_abs, i_off + (uint32_t)i), keys), tab);
    __nv_bfloat16* rowp = da + (tl * K + i) * 2 * d_ff;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t ch = blk * 128 + lane + 32 * j;
      if (ch < d_ff) {
        const float d = g.v[j];
        const float a = d * fmaf(d, fmaf(d, fmaf(d, c4[j], c3[j]), c2[j]), c1[j]);
        split_bf16(a, rowp + ch, rowp + d_ff + ch);
      }
    }
  }
}

// Down-projection draws: sigma eps on W_down's output (the block output h)
// is itself the head input change, dh = sigma eps, stored as bf16 hi/lo
// planes dh[row*2d + c], dh[row*2d + d + c]. One warp per (token, 128-channel
// block) walks the token's K draws, with the first two Philox rounds hoisted
// and the sigma-scaled table angle step.
__global__ __launch_bounds__(256) void k_mlp_noise_split(RoundKeys keys, uint32_t t_off,
                                                         uint32_t i_off, uint32_t ctr3,
                                                         float sigma, int64_t width, int32_t K,
                                                         int64_t t0, int64_t nt,
                                                         __nv_bfloat16* __restrict__ dh) {
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nblk = (width + 127) / 128;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= nt * nblk) return;  // no block-wide barrier follows
  const int64_t tl = wid / nblk;
  const int64_t blk = wid % nblk;
  const BlockConst bc = block_const(keys, slot_ctr0((uint32_t)blk, (uint32_t)lane), ctr3);
  const uint32_t t_abs = t_off + (uint32_t)(t0 + tl);
  for (int32_t i = 0; i < K; ++i) {
    const G4 g = gauss4_tab(philox_from2(bc, draw_const(keys, t_abs, i_off + (uint32_t)i), keys), tab);
    __nv_bfloat16* rowp = dh + (tl * K + i) * 2 * width;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t ch = blk * 128 + lane + 32 * j;
      if (ch < width) split_bf16(g.v[j], rowp + ch, rowp + width + ch);
    }
  }
}

// da = GELU(u + du) - GELU(u) for rows (token, draw) with du varying per
// element (the attention output-projection variant: du = sigma eps W_up^T).
// One warp per (token, 128-channel block) forms the Taylor coefficients of
// GELU at its channels' u once (as the up-projection kernel above) and walks
// the token's draws; the expansion serves |du| <= 1/16 (remainder < 2.3e-8),
// the quadrature form (gelu_delta) the rare larger du.
__global__ __launch_bounds__(256) void k_gelu_delta_rows(int64_t d_ff, int32_t K,
                                                         const float* __restrict__ u,
                                                         const float* __restrict__ du, int64_t t0,
                                                         int64_t nt,
                                                         __nv_bfloat16* __restrict__ da) {
  const int lane = threadIdx.x & 31;
  const int64_t nblk = (d_ff + 127) / 128;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= nt * nblk) return;
  const int64_t tl = wid / nblk;
  const int64_t blk = wid % nblk;
  const int64_t t = t0 + tl;
  float uu[4], c1[4], c2[4], c3[4], c4[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t ch = blk * 128 + lane + 32 * j;
    uu[j] = ch < d_ff ? u[t * d_ff + ch] : 0.0f;
    const double x = (double)uu[j];
    const double phi = 0.3989422804014327 * exp(-0.5 * x * x);
    const double Phi = 0.5 * erfc(-x * 0.7071067811865476);
    const double x2 = x * x;
    c1[j] = (float)(Phi + x * phi);
    c2[j] = (float)(phi * (2.0 - x2) * 0.5);
    c3[j] = (float)(phi * x * (x2 - 4.0) * (1.0 / 6.0));
    c4[j] = (float)(phi * (7.0 * x2 - x2 * x2 - 4.0) * (1.0 / 24.0));
  }
  // draws in groups of 4: the group's du loads are issued together, so each
  // warp keeps 16 loads in flight (the kernel streams du from HBM)
  constexpr int G = 4;
  for (int32_t i0 = 0; i0 < K; i0 += G) {
    float dd[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t ch = blk * 128 + lane + 32 * j;
        dd[g][j] = (i0 + g < K && ch < d_ff) ? du[(tl * K + i0 + g) * d_ff + ch] : 0.0f;
      }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (i0 + g >= K) break;
      __nv_bfloat16* rowp = da + (tl * K + i0 + g) * 2 * d_ff;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t ch = blk * 128 + lane + 32 * j;
        if (ch < d_ff) {
          const float x = dd[g][j];
          float a;
          if (fabsf(x) <= 0.0625f)
            a = x * fmaf(x, fmaf(x, fmaf(x, c4[j], c3[j]), c2[j]), c1[j]);
          else
            a = gelu_delta(uu[j], x);
          split_bf16(a, rowp + ch, rowp + d_ff + ch);
        }
      }
    }
  }
}

// a = GELU(u) in fp64, rounded once to fp32 (the down-projection's input,
// the right-hand operand of its weight gradient).
__global__ void k_gelu_f32(const float* __restrict__ u, int64_t n, float* __restrict__ a) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    a[i] = (float)gelu64((double)u[i]);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

constexpr int BM = 128, BN = 128, BKT = 16, PAD = 4;

// dz tile = dh (rows x d) . W_head^T, fused reward epilogue: per row and
// 128-column tile, sum_n p[t(row), n] expm1(dz) -> part[row * nparts + tile];
// dz at the target column -> dzy[row].
template <typename TI>
__global__ __launch_bounds__(256) void k_reward_gemm_simt(GemmDesc g, const float* __restrict__ P,
                                                          const int32_t* __restrict__ y,
                                                          int64_t t0, int32_t K,
                                                          float* __restrict__ part,
                                                          float* __restrict__ dzy) {
  __shared__ __align__(16) float As[BKT][BM + PAD];
  __shared__ __align__(16) float Bs[BKT][BN + PAD];
  const TI* A = (const TI*)g.A;
  const TI* B = (const TI*)g.B;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int64_t n0 = (int64_t)blockIdx.x * BN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int tid = threadIdx.x;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int64_t k0 = 0; k0 < g.K; k0 += BKT) {
    {
      const int r = tid >> 1, kk0 = (tid & 1) * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int64_t k = k0 + kk0 + q;
        const int64_t ma = m0 + r, nb = n0 + r;
        As[kk0 + q][r] = (ma < g.M && k < g.K) ? to_f(A[ma * g.lda + k]) : 0.0f;
        Bs[kk0 + q][r] = (nb < g.N && k < g.K) ? to_f(B[nb * g.ldb + k]) : 0.0f;
      }
    }
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
  const int64_t nparts = (g.N + BN - 1) / BN;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    const bool mrow = m < g.M;
    const int64_t t = t0 + (mrow ? m / K : 0);
    int32_t yt = mrow ? y[t] : -1;
    if (yt < 0 || (int64_t)yt >= g.N) yt = 0;  // reported by the loss kernel
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (mrow && n < g.N) {
        s = fmaf(P[t * g.N + n], expm1f(acc[i][j]), s);
        if (n == yt) dzy[m] = acc[i][j];
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (mrow && tx == 0) part[m * nparts + blockIdx.x] = s;
  }
}

__global__ void k_reward_combine_rows(const float* __restrict__ part, int nparts,
                                      const float* __restrict__ dzy, int64_t rows, int64_t row0,
                                      float* __restrict__ r) {
  const int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= rows) return;
  float s = 0.0f;
  for (int q = 0; q < nparts; ++q) s += part[m * nparts + q];
  r[row0 + m] = dzy[m] - log1pf(s);
}

// g_t[c] = scale * sum_i r[t*K + i] eps(t, i, c). A warp takes up to
// kNoiseGBlocks 128-channel blocks of one token (a unit), so the first two
// Philox rounds of a draw are formed once for all of them (those of a block
// once per unit); the table angle step (unit noise); the sums over draws in
// packed fp32x2 arithmetic (each lane rounds as fma(r, eps, acc) in draw
// order). A CTA holds 8 units, each warp staging its token's rewards.
constexpr int kNoiseGBlocks = 4;
constexpr int kNoiseGChunk = 256;  // rewards staged per warp at a time

template <typename TO>
__global__ __launch_bounds__(256) void k_noise_g(RoundKeys keys, uint32_t t_off, uint32_t i_off,
                                                 uint32_t ctr3, float scale, int64_t T,
                                                 int64_t width, int32_t K,
                                                 const float* __restrict__ r,
                                                 float* __restrict__ g_out, TO* __restrict__ gop,
                                                 int64_t plane) {
  __shared__ float rs[8][kNoiseGChunk];
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, 1.0f);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nblk = (width + 127) / 128;
  const int64_t ngroups = (nblk + kNoiseGBlocks - 1) / kNoiseGBlocks;
  const int64_t unit = (int64_t)blockIdx.x * 8 + warp;
  if (unit >= T * ngroups) return;  // no block-wide barrier follows
  const int64_t t = unit / ngroups;
  const int64_t blk0 = (unit % ngroups) * kNoiseGBlocks;
  const int nvalid = (int)min((int64_t)kNoiseGBlocks, nblk - blk0);
  const uint32_t t_abs = t_off + (uint32_t)t;
  BlockConst bc[kNoiseGBlocks];
  float2 a02[kNoiseGBlocks], a13[kNoiseGBlocks];
#pragma unroll
  for (int b = 0; b < kNoiseGBlocks; ++b) {
    bc[b] = block_const(keys, slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), ctr3);
    a02[b] = make_float2(0.f, 0.f);
    a13[b] = make_float2(0.f, 0.f);
  }
  for (int i0 = 0; i0 < K; i0 += kNoiseGChunk) {
    const int n = min(kNoiseGChunk, K - i0);
    __syncwarp();
    for (int q = lane; q < n; q += 32) rs[warp][q] = r[t * K + i0 + q];
    __syncwarp();
    for (int ii = 0; ii < n; ++ii) {
      const DrawConst dc = draw_const(keys, t_abs, i_off + (uint32_t)(i0 + ii));
      const float ri = rs[warp][ii];
      const float2 r2 = make_float2(ri, ri);
#pragma unroll
      for (int b = 0; b < kNoiseGBlocks; ++b) {
        if (b < nvalid) {
          const G4 g = gauss4_tab(philox_from2(bc[b], dc, keys), tab);
          a02[b] = __ffma2_rn(r2, make_float2(g.v[0], g.v[2]), a02[b]);
          a13[b] = __ffma2_rn(r2, make_float2(g.v[1], g.v[3]), a13[b]);
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kNoiseGBlocks; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t ch = (blk0 + b) * 128 + lane + 32 * j;
      if (b < nvalid && ch < width) {
        const float2 a = (j & 1) ? a13[b] : a02[b];
        const float v = ((j & 2) ? a.y : a.x) * scale;
        if (g_out) g_out[t * width + ch] = v;
        store_g_operand(gop, plane, t * width + ch, v);
      }
    }
}

}  // namespace

// k_noise_g geometry: T x (groups of kNoiseGBlocks 128-channel blocks) units,
// 8 per CTA of 256 threads.
struct NoiseGGeom {
  dim3 grid;
  unsigned threads;
};
static NoiseGGeom noise_g_geom(int64_t T, int64_t width) {
  const int64_t nblk = (width + 127) / 128;
  const int64_t units = T * ((nblk + kNoiseGBlocks - 1) / kNoiseGBlocks);
  return {dim3((unsigned)((units + 7) / 8)), 256u};
}

cudaError_t launch_mlp_delta_a(cudaStream_t st, const dust_params& p, const float* u, int64_t t0,
                               int64_t nt, __nv_bfloat16* da, bool round_bf16, float* da_f32) {
  if (round_bf16 && !da_f32 && p.sigma * 5.7686f <= 0.0625f) {
    const int64_t warps = nt * ((p.d_ff + 127) / 128);
    if (warps <= 0) return cudaSuccess;
    k_mlp_delta_a_taylor<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(
        round_keys(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
        ctr3_of(kTagMlpUp, p.stream_id), p.sigma, p.d_ff, p.K, u, t0, nt, da);
    return cudaGetLastError();
  }
  const int64_t rows = nt * p.K;
  const int64_t nblk = (p.d_ff + 127) / 128;
  const int64_t total = rows * nblk * 32;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  k_mlp_delta_a<<<(unsigned)((total + threads - 1) / threads), threads, 0, st>>>(
      key_of(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
      ctr3_of(kTagMlpUp, p.stream_id), p.sigma, p.d_ff, p.K, u, t0, rows,
      round_bf16 ? da : nullptr, da_f32);
  return cudaGetLastError();
}

cudaError_t launch_mlp_noise_split(cudaStream_t st, const dust_params& p, int64_t t0, int64_t nt,
                                   __nv_bfloat16* dh, int tag) {
  const int64_t warps = nt * ((p.d + 127) / 128);
  if (warps <= 0) return cudaSuccess;
  k_mlp_noise_split<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(
      round_keys(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset,
      ctr3_of(tag, p.stream_id), p.sigma, p.d, p.K, t0, nt, dh);
  return cudaGetLastError();
}

cudaError_t launch_gelu_delta_rows(cudaStream_t st, const dust_params& p, const float* u,
                                   const float* du, int64_t t0, int64_t nt, __nv_bfloat16* da) {
  const int64_t warps = nt * ((p.d_ff + 127) / 128);
  if (warps <= 0) return cudaSuccess;
  k_gelu_delta_rows<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p.d_ff, p.K, u, du, t0, nt, da);
  return cudaGetLastError();
}

cudaError_t launch_noise_g_planes(cudaStream_t st, const dust_params& p, const float* r,
                                  float* g_out, __nv_bfloat16* gop, int tag) {
  const NoiseGGeom gg = noise_g_geom(p.T, p.d);
  const float scale = p.sigma > 0.0f ? -1.0f / ((float)p.K * p.sigma) : 0.0f;
  k_noise_g<__nv_bfloat16><<<gg.grid, gg.threads, 0, st>>>(round_keys(p.seed), (uint32_t)p.token_offset,
      (uint32_t)p.draw_offset, ctr3_of(tag, p.stream_id), scale, p.T, p.d, p.K, r, g_out, gop,
      p.T * p.d);
  return cudaGetLastError();
}

cudaError_t launch_noise_g_f32(cudaStream_t st, const dust_params& p, const float* r,
                              float* g_out, float* gop, int tag) {
  const NoiseGGeom gg = noise_g_geom(p.T, p.d);
  const float scale = p.sigma > 0.0f ? -1.0f / ((float)p.K * p.sigma) : 0.0f;
  k_noise_g<float><<<gg.grid, gg.threads, 0, st>>>(round_keys(p.seed), (uint32_t)p.token_offset,
      (uint32_t)p.draw_offset, ctr3_of(tag, p.stream_id), scale, p.T, p.d, p.K, r, g_out, gop, 0);
  return cudaGetLastError();
}

cudaError_t launch_gelu_f32(cudaStream_t st, const float* u, int64_t n, float* a, int sm_count) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)sm_count * 16) blocks = (int64_t)sm_count * 16;
  k_gelu_f32<<<(unsigned)blocks, 256, 0, st>>>(u, n, a);
  return cudaGetLastError();
}

cudaError_t launch_reward_gemm_simt(cudaStream_t st, const GemmDesc& g, const float* P,
                                    const int32_t* y, int64_t t0, int32_t K, float* part,
                                    float* dzy) {
  dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM));
  if (g.dtype == DUST_BF16)
    k_reward_gemm_simt<__nv_bfloat16><<<grid, 256, 0, st>>>(g, P, y, t0, K, part, dzy);
  else
    k_reward_gemm_simt<float><<<grid, 256, 0, st>>>(g, P, y, t0, K, part, dzy);
  return cudaGetLastError();
}

cudaError_t launch_reward_combine_rows(cudaStream_t st, const float* part, int nparts,
                                       const float* dzy, int64_t rows, int64_t row0, int32_t K,
                                       float* r) {
  (void)K;
  const int threads = 256;
  k_reward_combine_rows<<<(unsigned)((rows + threads - 1) / threads), threads, 0, st>>>(
      part, nparts, dzy, rows, row0, r);
  return cudaGetLastError();
}

// a . b over n entries of a bf16 row and an fp32 row, this lane's share of it
// (the caller sums the warp). 16-byte loads where n is a multiple of 8: the
// callers' rows then start 16-byte aligned (allocation-aligned bases, row
// strides that are multiples of n).
__device__ __forceinline__ float warp_dot_bf16_f32(const __nv_bfloat16* __restrict__ a,
                                                   const float* __restrict__ b, int64_t n,
                                                   int lane) {
  float s = 0.0f;
  if ((n & 7) == 0) {
    for (int64_t i = (int64_t)lane * 8; i < n; i += 256) {
      const uint4 av = *reinterpret_cast<const uint4*>(a + i);
      const float4 b0 = *reinterpret_cast<const float4*>(b + i);
      const float4 b1 = *reinterpret_cast<const float4*>(b + i + 4);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&av);
      const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 af = __bfloat1622float2(a2[q]);
        s = fmaf(af.x, bb[2 * q], s);
        s = fmaf(af.y, bb[2 * q + 1], s);
      }
    }
  } else {
    for (int64_t i = lane; i < n; i += 32) s = fmaf(__bfloat162float(a[i]), b[i], s);
  }
  return s;
}

// First-order correction of the rewards for the lo plane of dh (the head GEMM
// contracts the hi plane only), and for the lo plane of da where dh came from
// its hi plane: a warp per (token, draw) row, 16-byte loads where the row
// lengths are multiples of 8.
__global__ __launch_bounds__(256) void k_mlp_reward_corr(const __nv_bfloat16* __restrict__ dh,
                                                         int64_t d, const float* __restrict__ Ut,
                                                         const __nv_bfloat16* __restrict__ da,
                                                         int64_t dff,
                                                         const float* __restrict__ Wv, int64_t t0,
                                                         int32_t K, int64_t rows,
                                                         float* __restrict__ r) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t t = t0 + row / K;
  float s = warp_dot_bf16_f32(dh + row * 2 * d + d, Ut + t * d, d, lane);
  if (da) s += warp_dot_bf16_f32(da + row * 2 * dff + dff, Wv + t * dff, dff, lane);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) r[t0 * K + row] += s;
}

// U_t := W_head[y_t] - U_t in place (T x d), and its bf16 copy.
__global__ void k_head_ut(const __nv_bfloat16* __restrict__ Wh, int64_t V,
                          const int32_t* __restrict__ y, float* __restrict__ U, int64_t T,
                          int64_t d, __nv_bfloat16* __restrict__ Ub) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T * d;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / d;
    int32_t yt = y[t];
    if (yt < 0 || (int64_t)yt >= V) yt = 0;  // reported by the loss kernel
    const float v = __bfloat162float(Wh[(int64_t)yt * d + (i - t * d)]) - U[i];
    U[i] = v;
    if (Ub) Ub[i] = __float2bfloat16_rn(v);
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ x, int64_t n,
                              __nv_bfloat16* __restrict__ out) {
  const int64_t n4 = n / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out + 4 * i);
    o[0] = __floats2bfloat162_rn(v.x, v.y);
    o[1] = __floats2bfloat162_rn(v.z, v.w);
  }
  for (int64_t i = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(x[i]);
}

cudaError_t launch_mlp_reward_corr(cudaStream_t st, const __nv_bfloat16* dh, int64_t d,
                                   const float* Ut, const __nv_bfloat16* da, int64_t dff,
                                   const float* Wv, int64_t t0, int32_t K, int64_t rows, float* r) {
  if (rows <= 0) return cudaSuccess;
  k_mlp_reward_corr<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(dh, d, Ut, da, dff, Wv, t0, K,
                                                                 rows, r);
  return cudaGetLastError();
}

cudaError_t launch_head_ut(cudaStream_t st, const __nv_bfloat16* W_head, int64_t V,
                           const int32_t* y, float* U, int64_t T, int64_t d, __nv_bfloat16* Ub,
                           int sm_count) {
  if (T * d <= 0) return cudaSuccess;
  int64_t blocks = (T * d + 255) / 256;
  if (blocks > (int64_t)sm_count * 16) blocks = (int64_t)sm_count * 16;
  k_head_ut<<<(unsigned)blocks, 256, 0, st>>>(W_head, V, y, U, T, d, Ub);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(cudaStream_t st, const float* x, int64_t n, __nv_bfloat16* out,
                               int sm_count) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n / 4 + 255) / 256;
  if (blocks > (int64_t)sm_count * 16) blocks = (int64_t)sm_count * 16;
  if (blocks < 1) blocks = 1;
  k_f32_to_bf16<<<(unsigned)blocks, 256, 0, st>>>(x, n, out);
  return cudaGetLastError();
}

cudaError_t launch_mlp_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                         void* gop, bool down) {
  const int64_t width = down ? p.d : p.d_ff;
  const NoiseGGeom gg = noise_g_geom(p.T, width);
  const float scale = p.sigma > 0.0f ? -1.0f / ((float)p.K * p.sigma) : 0.0f;
  const RoundKeys keys = round_keys(p.seed);
  const uint32_t c3 = ctr3_of(down ? kTagMlpDown : kTagMlpUp, p.stream_id);
  const int64_t plane = p.T * width;
  if (p.dtype == DUST_BF16 && !down)
    k_noise_g<__nv_bfloat16><<<gg.grid, gg.threads, 0, st>>>(keys, (uint32_t)p.token_offset,
        (uint32_t)p.draw_offset, c3, scale, p.T, width, p.K, r, g_out, (__nv_bfloat16*)gop, plane);
  else
    k_noise_g<float><<<gg.grid, gg.threads, 0, st>>>(keys, (uint32_t)p.token_offset,
        (uint32_t)p.draw_offset, c3, scale, p.T, width, p.K, r, g_out, (float*)gop, plane);
  return cudaGetLastError();
}

}  // namespace dust
