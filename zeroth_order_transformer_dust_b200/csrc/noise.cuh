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

// (float)i for |i| < 2^22, exactly, by exponent-bias arithmetic on the ALU
// pipe: 1.5 * 2^23 + i has i in its low mantissa bits.
__device__ __forceinline__ float small_int_to_float(int i) {
  return __int_as_float(0x4B400000 + i) - 12582912.0f;
}

// -ln(u) for u in (0, 1], accurate to a few ulp relative to the result,
// including u -> 1. u = 2^e m with m in [sqrt(1/2), sqrt(2)): subtracting the
// bit pattern of sqrt(1/2) before extracting the exponent lands m in that
// range without a branch. ln m is 2 atanh(s), s = (m-1)/(m+1), |s| <= 0.1716,
// from its Taylor series 2 s (1 + s^2/3 + s^4/5 + s^6/7) (truncation below
// 3e-8 absolute, vanishing as m -> 1); e ln 2 uses ln 2 split in a high part
// with 8 trailing zero bits (exact products for |e| <= 2^8) and a low
// correction (Cody and Waite's argument reduction).
__device__ __forceinline__ float neg_log_unit(float u) {
  const int bits = __float_as_int(u);
  const int e = (bits - 0x3f3504f3) >> 23;  // arithmetic shift: floor
  const float m = __int_as_float(bits - (e << 23));
  const float f = m - 1.0f;  // exact (Sterbenz)
  const float s = __fdividef(f, m + 1.0f);
  const float w = s * s;
  float poly = fmaf(w, 2.0f / 7.0f, 2.0f / 5.0f);
  poly = fmaf(w, poly, 2.0f / 3.0f);
  poly = fmaf(w, poly, 2.0f);
  const float ln_m = s * poly;
  const float fe = small_int_to_float(e);
  const float kLn2Hi = 0.693145751953125f;        // 0x3f317200
  const float kLn2Lo = 1.428606765330187e-06f;    // ln 2 - kLn2Hi
  const float ln_u = fmaf(fe, kLn2Hi, fmaf(fe, kLn2Lo, ln_m));
  return -ln_u;
}

// -ln(j 2^-24) for an integer j in [1, 2^24], the same computation as
// neg_log_unit with the 2^-24 scale folded into the exponent (the float of j
// is exact, and e - 24 comes out of the same exponent-bias subtraction).
__device__ __forceinline__ float neg_log_u24(uint32_t j) {
  const int bits = __float_as_int((float)j);
  const int e = (bits - 0x3f3504f3) >> 23;
  const float m = __int_as_float(bits - (e << 23));
  const float f = m - 1.0f;  // exact (Sterbenz)
  const float s = __fdividef(f, m + 1.0f);
  const float w = s * s;
  float poly = fmaf(w, 2.0f / 7.0f, 2.0f / 5.0f);
  poly = fmaf(w, poly, 2.0f / 3.0f);
  poly = fmaf(w, poly, 2.0f);
  const float ln_m = s * poly;
  const float fe = __int_as_float(0x4B400000 + e) - 12582936.0f;  // e - 24, exact
  const float kLn2Hi = 0.693145751953125f;
  const float kLn2Lo = 1.428606765330187e-06f;
  return -fmaf(fe, kLn2Hi, fmaf(fe, kLn2Lo, ln_m));
}

// sqrt(x) for x >= 0: the hardware reciprocal-square-root estimate y refined
// by one Newton-Raphson step on r = x y (r' = r + (y/2)(x - r^2)), which
// leaves about one ulp of error. x is clamped away from 0 (sqrt(0) -> 1e-15).
__device__ __forceinline__ float sqrt_newton(float x) {
  const float xs = fmaxf(x, 1e-30f);
  const float y = rsqrtf(xs);
  const float r = xs * y;
  const float e = fmaf(-r, r, xs);
  return fmaf(0.5f * y, e, r);
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

// Box-Muller on 24-bit uniforms: u1 = ((wa>>8)+1) 2^-24, u2 = (wb>>8) 2^-24;
// returns scale * (R cos 2 pi u2, R sin 2 pi u2), R = sqrt(-2 ln u1).
__device__ __forceinline__ float2 box_muller(uint32_t wa, uint32_t wb, float scale = 1.0f) {
  const float u1 = (float)((wa >> 8) + 1u) * 5.9604645e-08f;  // exact
  const float radius = scale * sqrt_newton(2.0f * neg_log_unit(u1));
  float s, c;
  sincos_turn24(wb >> 8, &s, &c);
  return make_float2(radius * c, radius * s);
}

// Table-driven variant of the angle step, for kernels that keep a 1024-entry
// table of roots of unity, tab[k] = (cos 2 pi k/1024, sin 2 pi k/1024), in
// shared memory: the angle 2 pi m 2^-24 is split into the nearest table angle
// plus a remainder |x| <= pi/1024, and cos/sin follow from the angle-addition
// formulas with cos x = 1 - x^2/2 and sin x = x (truncation below 5e-9).
constexpr int kSinCosTable = 1024;
constexpr int kSinCosTableAlloc = kSinCosTable + 1;  // entry 1024 repeats entry 0

__device__ __forceinline__ void fill_sincos_table(float2* tab) {
  for (int k = threadIdx.x; k < kSinCosTableAlloc; k += blockDim.x) {
    float s, c;
    sincospif((float)(k & (kSinCosTable - 1)) * (2.0f / kSinCosTable), &s, &c);
    tab[k] = make_float2(c, s);
  }
}

__device__ __forceinline__ void sincos_turn24_tab(uint32_t m, const float2* tab, float* s_out,
                                                  float* c_out) {
  const uint32_t idx = (m + (1u << 13)) >> 14;             // nearest 1/1024 turn, 0..1024
  const int r = (int)m - (int)(idx << 14);                  // [-2^13, 2^13)
  const float x = small_int_to_float(r) * 3.7450702e-07f;   // 2 pi / 2^24
  const float h = 0.5f * x * x;
  const float2 t = tab[idx];
  *c_out = fmaf(-t.y, x, fmaf(-t.x, h, t.x));
  *s_out = fmaf(t.x, x, fmaf(-t.y, h, t.y));
}

__device__ __forceinline__ float2 box_muller_tab(uint32_t wa, uint32_t wb, float scale,
                                                 const float2* tab) {
  const float radius = scale * sqrt_newton(2.0f * neg_log_u24((wa >> 8) + 1u));
  float s, c;
  sincos_turn24_tab(wb >> 8, tab, &s, &c);
  return make_float2(radius * c, radius * s);
}

// Four Gaussians of one counter (times `scale`): element j is output word j.
struct G4 {
  float v[4];
};

__device__ __forceinline__ G4 gauss4_tab(U4 w, float scale, const float2* tab) {
  const float2 a = box_muller_tab(w.x, w.y, scale, tab);
  const float2 b = box_muller_tab(w.z, w.w, scale, tab);
  G4 g;
  g.v[0] = a.x;
  g.v[1] = a.y;
  g.v[2] = b.x;
  g.v[3] = b.y;
  return g;
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

// Degree of expm1_small for noise of scale sigma (|eps| <= sqrt(48 ln 2) = 5.7686).
__host__ __device__ inline int expm1_degree(float sigma) {
  const float xmax = sigma * 5.7686f;
  if (xmax <= 0.03f) return 3;
  if (xmax <= 0.06f) return 4;
  return 0;
}

}  // namespace dust
