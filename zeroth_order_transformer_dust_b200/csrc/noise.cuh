// Counter-based Gaussian noise for the estimator, generated in registers.
//
// The Dust pages fix only that the noise is Gaussian and independent per
// token and per draw ("Dust：无需反向传播的Transformer零阶预训练", §1,
// 激活空间扰动). This build draws it from Philox4x32-10 (Salmon et al.,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) and Box-Muller on
// 24-bit uniforms; the slot -> (counter, word) layout puts the four words of
// one counter on slots l, l+32, l+64, l+96 of a 128-slot block so that a warp
// lane owns four coalesced columns per call.
#pragma once
#include <cstdint>

namespace dust {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

constexpr int kTagHead = 0;
constexpr int kTagSubsetOffset = 1;
constexpr int kTagMlpUp = 2;
constexpr int kTagMlpDown = 3;
constexpr int kTagAttnOut = 4;
constexpr int kTagAttnQ = 5;  // + 1: key, + 2: value
constexpr int kTagAttnK = 6;
constexpr int kTagAttnV = 7;

struct U4 {
  uint32_t x, y, z, w;
};

__host__ __device__ __forceinline__ uint32_t ctr3_of(int tag, uint32_t stream_id) {
  return (uint32_t)(tag & 0xff) | (stream_id << 8);
}

// One Philox round: two 32x32->64 products, hi/lo halves recombined with XOR.
__device__ __forceinline__ U4 philox_round(U4 c, uint32_t k0, uint32_t k1) {
  const uint64_t p0 = (uint64_t)kPhiloxM0 * c.x;
  const uint64_t p1 = (uint64_t)kPhiloxM1 * c.z;
  U4 o;
  o.x = (uint32_t)(p1 >> 32) ^ c.y ^ k0;
  o.y = (uint32_t)p1;
  o.z = (uint32_t)(p0 >> 32) ^ c.w ^ k1;
  o.w = (uint32_t)p0;
  return o;
}

// Philox4x32-10: ten rounds, key bumped between rounds.
__device__ __forceinline__ U4 philox10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    c = philox_round(c, k0, k1);
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
  return c;
}

// cos and sin of 2 pi m 2^-24 for an integer m in [0, 2^24). The nearest
// quarter turn is removed exactly in integer arithmetic, leaving
// |x| <= pi/4, where the Taylor series of sin (to x^9) and cos (to x^8) are
// truncated below 3e-8.
__device__ __forceinline__ void sincos_turn24(uint32_t m, float* s_out, float* c_out) {
  const uint32_t q = (m + (1u << 21)) >> 22;          // 0..4
  const int r = (int)m - (int)(q << 22);               // [-2^21, 2^21)
  const float x = (float)r * 3.7450702e-07f;           // 2 pi / 2^24
  const float x2 = x * x;
  float sp = fmaf(x2, 2.7557319e-06f, -1.9841270e-04f);  // 1/9!, -1/7!
  sp = fmaf(x2, sp, 8.3333333e-03f);                      // 1/5!
  sp = fmaf(x2, sp, -1.6666667e-01f);                     // -1/3!
  const float sn = fmaf(x * x2, sp, x);
  float cp = fmaf(x2, 2.4801587e-05f, -1.3888889e-03f);  // 1/8!, -1/6!
  cp = fmaf(x2, cp, 4.1666668e-02f);                      // 1/4!
  cp = fmaf(x2, cp, -0.5f);
  const float cs = fmaf(x2, cp, 1.0f);
  const uint32_t qq = q & 3u;
  float c = (qq & 1u) ? sn : cs;
  float s = (qq & 1u) ? cs : sn;
  c = (qq == 1u || qq == 2u) ? -c : c;
  s = (qq >= 2u) ? -s : s;
  *s_out = s;
  *c_out = c;
}

// Radius of the Box-Muller pair, R = sqrt(-2 ln u1), for
// u1 = ((wa >> 8) + 1) 2^-24 (exact in fp32), carried as
// rho = R / sqrt(2 ln 2) = sqrt(-log2 u1): the constant sqrt(2 ln 2) is
// folded into the angle table (or into the caller's scale) instead of
// costing a multiply per pair. Away from u1 = 1, log2 u1 is the hardware
// base-2 logarithm (MUFU.LG2). Its error near u1 = 1 is absolute (about
// 2^-23), which the square root turns into an error of about 0.5 2^-23 / rho,
// so for v = 1 - u1 < 2^-6 (exact; R < 0.18) the series
// -log2(1 - v) = (v + v^2/2 + v^3/3 + ...) / ln 2 is used instead (the first
// omitted term is below 2^-19 relative there). The square root is the
// hardware approximation (MUFU.SQRT, sqrt(0) = 0). Checked over all 2^24
// values of u1 against fp64.
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// base-2 logarithm (MUFU.LG2) for normal arguments: u1 >= 2^-24, so the
// flush-to-zero form needs no subnormal fix-up
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kRhoToR = 1.1774100f;  // sqrt(2 ln 2)

__device__ __forceinline__ float bm_rho(uint32_t wa) {
  const float u = fmaf((float)(wa >> 8), 5.9604645e-08f, 5.9604645e-08f);  // exact
  const float v = 1.0f - u;  // exact (u >= 1/2 where it is used)
  // log2(1 - v) = -(v + v^2/2 + v^3/3) / ln 2, truncated
  const float near = v * fmaf(v, fmaf(v, -0.48089835f, -0.7213475f), -1.442695f);
  return sqrt_approx(-(v < 0.015625f ? near : lg2_approx(u)));
}

// Box-Muller on 24-bit uniforms: u1 = ((wa>>8)+1) 2^-24, u2 = (wb>>8) 2^-24;
// returns scale * (R cos 2 pi u2, R sin 2 pi u2), R = sqrt(-2 ln u1).
__device__ __forceinline__ float2 box_muller(uint32_t wa, uint32_t wb, float scale = 1.0f) {
  const float radius = (scale * kRhoToR) * bm_rho(wa);
  float s, c;
  sincos_turn24(wb >> 8, &s, &c);
  return make_float2(radius * c, radius * s);
}

// Table-driven variant of the angle step, for kernels that keep 1024 roots of
// unity at interval midpoints, theta_k = 2 pi (k + 1/2) / 1024, in shared
// memory, already scaled by sigma sqrt(2 ln 2) (the radius factor that
// bm_rho leaves out): tab[k] = sigma sqrt(2 ln 2) (cos theta_k, sin theta_k).
// The 24-bit angle m = wb >> 8 is interval wb >> 22 plus the remainder
// x = c xr, c = 2 pi 2^-32, xr = (r - 2^13) 2^8 with r bits 8..21 of wb
// (|x| <= pi/1024). The float F = 1.5 2^23 + r 2^8 comes exactly from an
// exponent-bias construction and x = fma(F, c, -(1.5 2^23 + 2^21) c) in one
// rounding (the rounded constant moves x by under 1e-9). cos/sin follow from
// the angle-addition formulas with cos x = 1 - x^2/2 and sin x = x
// (truncation below 5e-9). Checked over all 2^24 angles (sigma = 1) against
// sqrt(2 ln 2) (cos, sin) in fp64.
constexpr int kSinCosTable = 1024;

__device__ __forceinline__ void fill_sincos_table(float2* tab, float sigma) {
  const float scale = sigma * kRhoToR;
  for (int k = threadIdx.x; k < kSinCosTable; k += blockDim.x) {
    float s, c;
    sincospif((float)(2 * k + 1) * (1.0f / kSinCosTable), &s, &c);
    tab[k] = make_float2(scale * c, scale * s);
  }
}

// sigma sqrt(2 ln 2) (cos, sin) of the angle of word wb.
__device__ __forceinline__ float2 rotate_tab(uint32_t wb, const float2* tab) {
  const float F = __int_as_float((wb & 0x003FFF00u) | 0x4B400000u);
  const float x = fmaf(F, 1.4629181e-09f, -0.021475732f);  // c = 2 pi 2^-32
  const float2 t = tab[wb >> 22];
  const float q = fmaf(x * x, -0.5f, 1.0f);
  return make_float2(fmaf(-t.y, x, t.x * q), fmaf(t.x, x, t.y * q));
}

__device__ __forceinline__ float2 box_muller_tab(uint32_t wa, uint32_t wb, const float2* tab) {
  const float rho = bm_rho(wa);
  const float2 cs = rotate_tab(wb, tab);
  return make_float2(rho * cs.x, rho * cs.y);
}

// Four Gaussians of one counter (times `scale`): element j is output word j.
struct G4 {
  float v[4];
};

__device__ __forceinline__ G4 gauss4_tab(U4 w, const float2* tab) {
  const float2 a = box_muller_tab(w.x, w.y, tab);
  const float2 b = box_muller_tab(w.z, w.w, tab);
  G4 g;
  g.v[0] = a.x;
  g.v[1] = a.y;
  g.v[2] = b.x;
  g.v[3] = b.y;
  return g;
}

// gauss4_tab with the two Box-Muller pairs of the counter, (w.x, w.y) and
// (w.z, w.w), computed side by side in packed fp32x2 arithmetic (one
// instruction per pair of operations; each lane of a packed operation rounds
// as the scalar one does): the same operations on the same values in the same
// order, so the results equal gauss4_tab's bit for bit. e02 holds words 0 and
// 2 (the cosine outputs of the two pairs), e13 words 1 and 3 (the sines).
__device__ __forceinline__ void gauss4_tab_x2(U4 w, const float2* tab, float2& e02, float2& e13) {
  const float2 k24 = make_float2(5.9604645e-08f, 5.9604645e-08f);
  const float2 u = __ffma2_rn(make_float2((float)(w.x >> 8), (float)(w.z >> 8)), k24, k24);
  const float2 v = __ffma2_rn(u, make_float2(-1.0f, -1.0f), make_float2(1.0f, 1.0f));  // 1 - u
  float2 near = __ffma2_rn(v, make_float2(-0.48089835f, -0.48089835f),
                           make_float2(-0.7213475f, -0.7213475f));
  near = __ffma2_rn(v, near, make_float2(-1.442695f, -1.442695f));
  near = __fmul2_rn(v, near);
  const float2 rho = make_float2(sqrt_approx(-(v.x < 0.015625f ? near.x : lg2_approx(u.x))),
                                 sqrt_approx(-(v.y < 0.015625f ? near.y : lg2_approx(u.y))));
  const float2 F = make_float2(__int_as_float((w.y & 0x003FFF00u) | 0x4B400000u),
                               __int_as_float((w.w & 0x003FFF00u) | 0x4B400000u));
  const float2 x = __ffma2_rn(F, make_float2(1.4629181e-09f, 1.4629181e-09f),
                              make_float2(-0.021475732f, -0.021475732f));
  const float2 nx = __ffma2_rn(F, make_float2(-1.4629181e-09f, -1.4629181e-09f),
                               make_float2(0.021475732f, 0.021475732f));  // -x, exactly
  const float2 q = __ffma2_rn(__fmul2_rn(x, x), make_float2(-0.5f, -0.5f), make_float2(1.0f, 1.0f));
  const float2 ta = tab[w.y >> 22], tb = tab[w.w >> 22];
  const float2 c = make_float2(ta.x, tb.x), s = make_float2(ta.y, tb.y);
  e02 = __fmul2_rn(rho, __ffma2_rn(s, nx, __fmul2_rn(c, q)));
  e13 = __fmul2_rn(rho, __ffma2_rn(c, x, __fmul2_rn(s, q)));
}

__device__ __forceinline__ G4 gauss4(U4 w, float scale = 1.0f) {
  const float2 a = box_muller(w.x, w.y, scale);
  const float2 b = box_muller(w.z, w.w, scale);
  G4 g;
  g.v[0] = a.x;
  g.v[1] = a.y;
  g.v[2] = b.x;
  g.v[3] = b.y;
  return g;
}

// log1p(s): short series for |s| < 2^-10 (truncation s^4/4 < 2^-42), the
// library function otherwise. Callers pass warp-uniform s.
__device__ __forceinline__ float log1p_small(float s) {
  if (fabsf(s) < 9.765625e-4f) return s * fmaf(s, fmaf(s, 1.0f / 3.0f, -0.5f), 1.0f);
  return log1pf(s);
}

// Round keys of a launch: rk0[r] = k0 + r 0x9E3779B9, rk1[r] = k1 + r 0xBB67AE85.
// Kernels take them as __grid_constant__ parameters so that the XORs read
// them from the constant bank.
struct RoundKeys {
  uint32_t rk0[10], rk1[10];
};

__host__ inline RoundKeys round_keys(uint64_t seed) {
  RoundKeys k;
  const uint32_t k0 = (uint32_t)(seed & 0xffffffffu), k1 = (uint32_t)(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    k.rk0[r] = k0 + (uint32_t)r * kPhiloxW0;
    k.rk1[r] = k1 + (uint32_t)r * kPhiloxW1;
  }
  return k;
}

// Philox4x32-10 with rounds 0 and 1 precomputed. Round 0 maps the counter
// (c0, t, i, c3) to (A, B, C, D), with A and B functions of the draw (t, i)
// and C, D of the slot block (c0, c3); round 1 maps that to
// (E ^ B, F, G ^ D', H), with E, F, D' per slot block and G, H per draw.
// A kernel that loops over draws for fixed slot blocks evaluates these once.
struct DrawConst {
  uint32_t B, G, H;
};
struct BlockConst {
  uint32_t E, F, Dp;
};

__device__ __forceinline__ BlockConst block_const(const RoundKeys& K, uint32_t c0, uint32_t c3) {
  const uint64_t p0 = (uint64_t)kPhiloxM0 * c0;
  const uint32_t C = (uint32_t)(p0 >> 32) ^ c3 ^ K.rk1[0];
  const uint32_t D = (uint32_t)p0;
  const uint64_t p1 = (uint64_t)kPhiloxM1 * C;
  BlockConst b;
  b.E = (uint32_t)(p1 >> 32) ^ K.rk0[1];
  b.F = (uint32_t)p1;
  b.Dp = D ^ K.rk1[1];
  return b;
}

__device__ __forceinline__ DrawConst draw_const(const RoundKeys& K, uint32_t t_abs, uint32_t i_abs) {
  const uint64_t p1 = (uint64_t)kPhiloxM1 * i_abs;
  const uint32_t a = (uint32_t)(p1 >> 32) ^ t_abs ^ K.rk0[0];
  DrawConst d;
  d.B = (uint32_t)p1;
  const uint64_t p0 = (uint64_t)kPhiloxM0 * a;
  d.G = (uint32_t)(p0 >> 32);
  d.H = (uint32_t)p0;
  return d;
}

__device__ __forceinline__ U4 philox_from2(const BlockConst& bc, const DrawConst& dc,
                                           const RoundKeys& K) {
  U4 c{bc.E ^ dc.B, bc.F, dc.G ^ bc.Dp, dc.H};
#pragma unroll
  for (int r = 2; r < 10; ++r) c = philox_round(c, K.rk0[r], K.rk1[r]);
  return c;
}

// Counter word 0 for slot block `blk` (128 slots) and lane `lane`.
__host__ __device__ __forceinline__ uint32_t slot_ctr0(uint32_t blk, uint32_t lane) {
  return (blk << 5) | lane;
}

// Key of a 64-bit seed.
struct Key {
  uint32_t k0, k1;
};
__host__ __device__ __forceinline__ Key key_of(uint64_t seed) {
  return Key{(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
}

// eps of one slot (generic path; the hot kernels generate a whole counter).
__device__ __forceinline__ float gauss_slot(Key key, uint32_t t_abs, uint32_t i_abs,
                                            uint32_t ctr3, uint32_t k) {
  U4 c{slot_ctr0(k >> 7, k & 31u), t_abs, i_abs, ctr3};
  const U4 w = philox10(c, key.k0, key.k1);
  const uint32_t word = (k >> 5) & 3u;
  const uint32_t wa = (word < 2) ? w.x : w.z;
  const uint32_t wb = (word < 2) ? w.y : w.w;
  const float2 n = box_muller(wa, wb);
  return (word & 1u) ? n.y : n.x;
}

// Subset offset b = floor(w0 V / 2^32) of (token, draw).
__device__ __forceinline__ uint32_t subset_offset(Key key, uint32_t t_abs, uint32_t i_abs,
                                                  uint32_t stream_id, uint32_t V) {
  U4 c{0u, t_abs, i_abs, ctr3_of(kTagSubsetOffset, stream_id)};
  const U4 w = philox10(c, key.k0, key.k1);
  return (uint32_t)(((uint64_t)w.x * V) >> 32);
}

// expm1 from its Taylor series of degree DEG (0: the library function). The
// callers form s = sum_j p_j expm1(x_j) with sum_j p_j <= 1, so a truncation
// |x|^(DEG+1)/(DEG+1)! bounds the absolute error of s: degree 3 for
// |x| <= 0.03 leaves < 3.4e-8, degree 4 for |x| <= 0.06 < 6.5e-9
// (expm1_degree picks DEG from sigma).
template <int DEG>
__device__ __forceinline__ float expm1_small(float x) {
  if constexpr (DEG == 3) {
    float q = fmaf(x, 1.0f / 6.0f, 0.5f);
    q = fmaf(x, q, 1.0f);
    return x * q;
  } else if constexpr (DEG == 4) {
    float q = fmaf(x, 1.0f / 24.0f, 1.0f / 6.0f);
    q = fmaf(x, q, 0.5f);
    q = fmaf(x, q, 1.0f);
    return x * q;
  } else if constexpr (DEG == 5) {
    float q = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
    q = fmaf(x, q, 1.0f / 6.0f);
    q = fmaf(x, q, 0.5f);
    q = fmaf(x, q, 1.0f);
    return x * q;
  } else {
    return expm1f(x);
  }
}

// expm1_small of a pair, in packed fp32x2 arithmetic (the same operations per
// lane as the scalar form).
template <int DEG>
__device__ __forceinline__ float2 expm1_small_x2(float2 x) {
  if constexpr (DEG == 3) {
    float2 q = __ffma2_rn(x, make_float2(1.0f / 6.0f, 1.0f / 6.0f), make_float2(0.5f, 0.5f));
    q = __ffma2_rn(x, q, make_float2(1.0f, 1.0f));
    return __fmul2_rn(x, q);
  } else if constexpr (DEG == 4) {
    float2 q = __ffma2_rn(x, make_float2(1.0f / 24.0f, 1.0f / 24.0f),
                          make_float2(1.0f / 6.0f, 1.0f / 6.0f));
    q = __ffma2_rn(x, q, make_float2(0.5f, 0.5f));
    q = __ffma2_rn(x, q, make_float2(1.0f, 1.0f));
    return __fmul2_rn(x, q);
  } else if constexpr (DEG == 5) {
    float2 q = __ffma2_rn(x, make_float2(1.0f / 120.0f, 1.0f / 120.0f),
                          make_float2(1.0f / 24.0f, 1.0f / 24.0f));
    q = __ffma2_rn(x, q, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
    q = __ffma2_rn(x, q, make_float2(0.5f, 0.5f));
    q = __ffma2_rn(x, q, make_float2(1.0f, 1.0f));
    return __fmul2_rn(x, q);
  } else {
    return make_float2(expm1f(x.x), expm1f(x.y));
  }
}

// Sum over the warp (all lanes get it) of values whose magnitudes add up to
// less than 2^-3: each rounded to 2^-34 fixed point, the integers added
// exactly by the warp-reduction unit (no overflow below 2^31), the sum scaled
// back. The rounding moves each lane's share by at most 2^-35.
__device__ __forceinline__ float warp_sum_fixed34(float v) {
  const int q = __float2int_rn(v * 17179869184.0f);  // 2^34
  return (float)__reduce_add_sync(0xffffffffu, q) * 5.8207661e-11f;  // 2^-34
}

// Degree of expm1_small for noise of scale sigma (|eps| <= sqrt(48 ln 2) = 5.7686).
__host__ __device__ inline int expm1_degree(float sigma) {
  const float xmax = sigma * 5.7686f;
  if (xmax <= 0.03f) return 3;
  if (xmax <= 0.06f) return 4;
  return 0;
}

}  // namespace dust
