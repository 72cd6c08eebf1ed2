// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <string>

#include "../../include/dust.h"

namespace dust {

// Bits of the device status word.
enum : uint32_t {
  kStatusBadTarget = 1u << 0,
  kStatusTimeout = 1u << 1,
  kStatusRange = 1u << 2,  // an operand outside the range a kernel's format holds
};

struct Buf {
  void* p = nullptr;
  size_t bytes = 0;
};

// Host helpers of the subset rule j_k = (a k + b) mod V, shared by every entry
// point that draws vocabulary subsets, so all of them pick the same stride.
inline int64_t gcd64(int64_t a, int64_t b) {
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  return a < 0 ? -a : a;
}

// Inverse of a modulo m (gcd(a, m) = 1), extended Euclid.
inline int64_t modinv(int64_t a, int64_t m) {
  if (m == 1) return 0;
  int64_t t = 0, nt = 1, r = m, nr = a % m;
  while (nr != 0) {
    const int64_t q = r / nr;
    int64_t tmp = t - q * nt;
    t = nt;
    nt = tmp;
    tmp = r - q * nr;
    r = nr;
    nr = tmp;
  }
  return t < 0 ? t + m : t;
}

// Default stride: the smallest integer >= V (sqrt 5 - 1) / 2 coprime to V.
int64_t default_stride(int64_t V);
// The stride a call uses: subset_a mod V when given, else default_stride(V).
inline int64_t subset_stride_of(const dust_params& p) {
  return p.subset_a ? p.subset_a % p.V : default_stride(p.V);
}

// Launch geometry of the GEMMs: A(m, k) and B(n, k) addressing.
struct GemmDesc {
  int64_t M, N, K;
  const void* A;
  int64_t lda;        // A(m,k) = A[m*lda + k] if a_kmajor, else A[k*lda + m]
  bool a_kmajor;
  const void* B;
  int64_t ldb;        // B(n,k) = B[n*ldb + k] if b_kmajor, else B[k*ldb + n]
  bool b_kmajor;
  int64_t b_row_mul;  // nonzero: B row n is source row (n * b_row_mul) mod N
  int dtype;          // DUST_F32 or DUST_BF16 for both operands
  bool f16 = false;   // with DUST_BF16: the 2-byte operands are fp16 instead
};

enum EpiKind {
  kEpiF32 = 0,         // C[mo*ldc + n] = acc, mo = (m*c_row_mul) mod M when c_row_mul != 0
  kEpiBF16 = 1,        // Cb[m*ldcb + n] = bf16(acc)
  kEpiGeluSplit = 2,   // C[m*ldc + n] = acc (u); a = GELU(acc) in fp64, stored as bf16
                       // hi/lo planes Cb[m*ldcb + n], Cb[m*ldcb + split + n]
  kEpiResidSplit = 3,  // h = resid[m*ldr + n] (bf16; plus resid[m*ldr + rsplit + n] when
                       // rsplit > 0, a hi/lo pair) + acc, stored as bf16 hi/lo planes
  kEpiSplit = 4,       // acc stored as bf16 hi/lo planes Cb[m*ldcb + n], Cb[m*ldcb + split + n]
  kEpiReward = 5,      // MLP perturbed logits dz (never stored): per row m, 256-column
                       // tile nb and 128-column half h, part[(m*n_tiles + nb)*2 + h] =
                       // sum_n P[t, n] expm1(dz); dzy[m] = dz at column y[t];
                       // t = t0 + m / draws
  kEpiF32Lse = 6,      // kEpiF32 without row remap, plus per row m, 256-column tile nb
                       // and half h the softmax partial lsep[(m*n_tiles + nb)*2 + h] =
                       // (max_n acc, sum_n exp(acc - max)) over its columns < N
};

struct EpiDesc {
  int kind = kEpiF32;
  float* C = nullptr;
  int64_t ldc = 0;
  __nv_bfloat16* Cb = nullptr;
  int64_t ldcb = 0;
  int64_t split = 0;
  int64_t c_row_mul = 0;
  const void* resid = nullptr;
  int64_t ldr = 0;
  int64_t rsplit = 0;
  // kEpiReward
  const float* P = nullptr;
  const int32_t* y = nullptr;
  int64_t t0 = 0;
  int32_t draws = 1;
  float* part = nullptr;
  float* dzy = nullptr;
  // kEpiF32Lse
  float2* lsep = nullptr;
  // kEpiF32: when set, every stored value is acc * (*scale) (a power of two
  // written on the device by the kernel that scaled the operands)
  const float* scale = nullptr;
};

// Column tile width of the tensor-core GEMM; its epilogues leave two partials
// per row and tile (tc_partials_per_row).
constexpr int kTcTileN = 256;
inline int tc_partials_per_row(int64_t N) { return (int)(2 * ((N + kTcTileN - 1) / kTcTileN)); }

// Exact-erf GELU in fp64. The last product is rounded on its own
// (__dmul_rn) so that a difference GELU(x) - GELU(x') is not contracted
// into a fused multiply-add: equal arguments then give an exact zero.
__device__ __forceinline__ double gelu64(double x) {
  return __dmul_rn(0.5 * x, 1.0 + erf(x * 0.70710678118654752440));
}

// v as a bf16 pair with v ~= hi + lo (relative error about 2^-17). For an
// fp32 v the residual v - hi is exact in fp32 (it has at most 16 significant
// bits), so the float form gives the same pair as the fp64 one.
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *hi = h;
  *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}
__device__ __forceinline__ void split_bf16(double v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn((float)v);
  *hi = h;
  *lo = __float2bfloat16_rn((float)(v - (double)__bfloat162float(h)));
}

// Round an fp64 value to the nearest bf16 (8 significant bits, ties to even)
// in one step: the mantissa is rounded on the fp64 bit pattern, after which the
// value is exactly representable in fp32 and bf16.
__device__ __forceinline__ __nv_bfloat16 bf16_from_f64(double v) {
  unsigned long long b = (unsigned long long)__double_as_longlong(v);
  const unsigned long long keep = (b >> 45) & 1ull;  // lowest kept mantissa bit
  b = (b + 0x00000FFFFFFFFFFFull + keep) & ~0x00001FFFFFFFFFFFull;
  return __float2bfloat16_rn((float)__longlong_as_double((long long)b));
}

// The bf16 GEMM operand of g is stored as two planes, hi = bf16(v) and
// lo = bf16(v - hi), `plane` elements apart, so sum_t g_t h_t^T computed over
// both planes carries about 2^-17 relative error from the operand instead of
// the 2^-9 of a single bf16 rounding.
__device__ __forceinline__ void store_g_operand(__nv_bfloat16* gop, int64_t plane, int64_t o,
                                                float v) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  gop[o] = hi;
  gop[plane + o] = __float2bfloat16_rn(v - __bfloat162float(hi));
}
__device__ __forceinline__ void store_g_operand(float* gop, int64_t, int64_t o, float v) {
  gop[o] = v;
}

// Formats of the g operand the LM-head draw kernels leave for the G_W GEMM.
// kGopF16: one fp16 plane holding g * scale, scale = 2^e chosen on the host
// from the bound the noise puts on g (head_gop_format), so every value is in
// range; its rounding (2^-11 relative) sits well inside the bf16 G_W
// tolerance and the GEMM contracts over T instead of the planes' 2T.
enum GopKind : int { kGopF32 = 0, kGopBf16Planes = 1, kGopF16 = 2 };
struct GopFormat {
  int kind;
  float scale;  // kGopF16 only
};
__device__ __forceinline__ void store_gop(void* gop, GopFormat f, int64_t plane, int64_t o,
                                          float v) {
  if (f.kind == kGopF16)
    ((__half*)gop)[o] = __float2half_rn(v * f.scale);
  else if (f.kind == kGopBf16Planes)
    store_g_operand((__nv_bfloat16*)gop, plane, o, v);
  else
    ((float*)gop)[o] = v;
}
// The format of the estimator call: fp32 for fp32 inputs, else kGopF16.
GopFormat head_gop_format(const dust_params& p);
// Bytes of a g operand of T x width in format f.
size_t gop_format_bytes(GopFormat f, int64_t T, int64_t width);

}  // namespace dust

struct dust_ctx {
  int device = 0;
  cudaStream_t stream = nullptr;
  int sm_count = 0;
  int max_smem_optin = 0;
  std::string last_error;
  uint32_t* d_status = nullptr;
  uint32_t* h_status = nullptr;  // pinned
  // stage timing (events recorded between the stages of a call)
  static constexpr int kMaxMarks = 16;
  bool timing = false;
  cudaEvent_t ev[kMaxMarks] = {};
  const char* mark_name[kMaxMarks] = {};
  int nmarks = 0;
  int64_t launches = 0;
  // tensor-core GEMMs on (DUST_DISABLE_TC=1 at creation routes all GEMMs to CUDA cores)
  bool tc_enabled = true;
  // CTA-pair tensor-core GEMMs for M >= 256 (DUST_TC_PAIR=0 at creation keeps one CTA per tile)
  bool tc_pair = true;
  // shared-memory subset kernel on (DUST_SUBSET_KERNEL=1 selects the first, L2-fed one)
  bool subset2_enabled = true;
  // full-vocabulary draws in one pass where a plan fits (DUST_FULL_KERNEL=2 at creation: two)
  bool full_one_enabled = true;
  // the two passes beside the one-pass kernel on the SMs its clusters leave empty
  // (DUST_FULL_SPLIT=0 at creation: off); their streams (high and low priority)
  // and the fork/join events are made at first use
  bool full_split = true;
  cudaStream_t side_hi = nullptr, side_lo = nullptr;
  cudaEvent_t fork_ev = nullptr, join_hi = nullptr, join_lo = nullptr;
  // scratch, grown on demand
  dust::Buf z, lse, loss, gop, rew, part, wperm, gT, hT, xdup, dzy, mlp_u, mlp_a, mlp_h, mlp_da,
      mlp_dh, wd2, wh2, in_h, in_w, in_y, out_g, out_loss, out_r, out_gv, lsep, mlp_a32, mlp_dn, mlp_du, wu2,
      attn_o, attn_lse, attn_gb, attn_w, attn_tcr, attn_coef,
      hsc,            // the fp16 G_W path's largest |h| and epilogue scale
      mlp_pb, mlp_uw,  // the MLP rewards' correction: P in bf16, U = P W_head,
      mlp_ub, mlp_wv,  // U in bf16, Wv = U W_down
      mlp_wt;          // W_head or W_down transposed for those GEMMs
};

namespace dust {

// Kernel launchers (all enqueue on `st`, return cudaGetLastError()).
cudaError_t launch_debug_philox(cudaStream_t st, uint64_t seed, const uint32_t* ctr, int64_t n,
                                uint32_t* out);
// method 0: polynomial angle step; 1: table-driven angle step in the packed
// fp32x2 form of the draw kernels; 2: the same step in scalar form.
cudaError_t launch_sgd_momentum(cudaStream_t st, int64_t n, float lr, float mu, const float* G,
                                float* v, float* W, __nv_bfloat16* Wb, int sm_count);
// what: 0 = radius for all 2^24 u1 (2^24 floats), 1 = polynomial angle step,
// 2 = table angle step (2 x 2^24 floats: cos, sin).
cudaError_t launch_debug_bm(cudaStream_t st, int what, float sigma, float* out);
cudaError_t launch_debug_gauss(cudaStream_t st, const dust_params& p, int tag, int64_t nt,
                               int64_t ni, int64_t nslots, float* out, int method);

cudaError_t launch_gemm_simt(cudaStream_t st, const GemmDesc& g, const EpiDesc& e);

// Row-wise log-sum-exp of Z (T x V). Writes lse[t], loss[t] = lse - Z[t, col(y_t)]
// with col(y) = y (col_mul == 0) or (y * col_mul) mod V; if to_prob, overwrites Z
// with exp(Z - lse). Sets kStatusBadTarget for targets outside [0, V).
// LSE and clean loss of each row from the clean GEMM's per-tile softmax
// partials (kEpiF32Lse), ntiles = ceil(V / kTcTileN) per row.
cudaError_t launch_lse_combine(cudaStream_t st, const float2* lsep, int ntiles, const float* Z,
                               int64_t T, int64_t V, const int32_t* y, int64_t col_mul,
                               float* lse, float* loss, uint32_t* status);
cudaError_t launch_lse_rows(cudaStream_t st, float* Z, int64_t T, int64_t V, const int32_t* y,
                            int64_t col_mul, float* lse, float* loss, bool to_prob,
                            uint32_t* status);

// Full-vocabulary reward, stage 1: partial sums sum_j p_j expm1(sigma eps_j) per
// (token, slab, draw) -> part[(t * nslab + slab) * K + i], and sigma eps at the
// target -> xy[t * K + i] (T x K floats, full_vocab_xy_bytes).
int full_vocab_nslab(int64_t V);
size_t full_vocab_xy_bytes(int64_t T, int32_t K);
// Where the two passes share the GPU with a one-pass launch (full_split_plan):
// their grids fill only `sms` SMs, each CTA with `pad` bytes of dynamic shared
// memory it does not use, so that none fits on an SM beside a one-pass CTA.
struct FullSide {
  int sms = 0;
  size_t pad = 0;
};
cudaError_t launch_full_reward_partial(cudaStream_t st, const dust_params& p, const float* Z,
                                       const float* lse,
                                       const int32_t* y, float* part, float* xy,
                                       const FullSide* side = nullptr);
// Stage 2: r[t*K + i] = xy - log1p(sum_slab part).
cudaError_t launch_full_reward_combine(cudaStream_t st, const dust_params& p, const float* part,
                                       const float* xy, float* r);
// Stage 3: g_t = -(1/(K sigma)) sum_i r_i eps_i; writes g (fp32, optional) and the
// GEMM operand gop in format gf.
cudaError_t launch_full_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                          void* gop, GopFormat gf, const FullSide* side = nullptr);

// Full-vocabulary draws in one pass (the noise generated once): clusters of nb
// CTAs (at most 4), one token row per cluster at a time, W generator warps and
// one reducer warp per CTA. full_one_plan returns false where no configuration
// fits (the three stages above run then).
struct FullOnePlan {
  int nb = 0, W = 0, ncl = 0;
  size_t smem = 0;
};
bool full_one_plan(const dust_params& p, int sm_count, int max_smem_optin, FullOnePlan* out);
// Rewards to r (T x K, may be null), g and the GEMM operand as launch_full_g; a
// wait that expires sets kStatusTimeout in *status.
cudaError_t launch_full_one(cudaStream_t st, const dust_params& p, const FullOnePlan& plan,
                            const float* Z, const float* lse, const int32_t* y, float* r,
                            float* g_out, void* gop, GopFormat gf, uint32_t* status);
// Tokens of a call that the two passes take from the end of the batch, on the
// SMs that `one`'s clusters leave empty and concurrently with the one-pass
// launch over the rest (which then fills `one.ncl` clusters a whole number of
// times); 0 where that does not pay. Fills *side.
int64_t full_split_plan(const dust_params& p, const FullOnePlan& one, int sm_count,
                        FullSide* side);

// Subset draws, fused reward + accumulation. P is the probability matrix in
// permuted column order (column q holds vocabulary index (a q) mod V).
// gacc: T x V fp32 accumulator, needed only when a row does not fit in
// shared memory (subset_gacc_bytes() > 0).
size_t subset_gacc_bytes(int64_t T, int64_t V, int max_smem_optin);
cudaError_t launch_subset_impl(cudaStream_t st, const dust_params& p, int64_t a, int64_t a_inv,
                               const float* P, const int32_t* y, float* rewards, float* g_out,
                               void* gop, GopFormat gf, float* gacc, int max_smem_optin);

// Subset draws with the probability row and the g accumulator resident in
// shared memory, one cluster of 1 to 8 CTAs per token (0: not applicable to
// this V, S). Z holds clean logits in permuted column order, lse the row
// log-sum-exp; p = exp(z - lse) is formed while the row is loaded. A row
// copy that does not arrive in time sets kStatusTimeout in *status.
int subset2_cluster_size(int64_t V, int32_t S, int max_smem_optin);
cudaError_t launch_subset2(cudaStream_t st, const dust_params& p, int64_t a, int64_t a_inv,
                           const float* Z, const float* lse, const int32_t* y, float* rewards,
                           float* g_out, void* gop, GopFormat gf, int max_smem_optin,
                           int sm_count, uint32_t* status);

// Tensor-core GEMM (tcgen05): shapes it takes, and its launcher (pair: a
// 256 x 256 tile per cluster of two CTAs, cta_group::2; else 128 x 256 per
// CTA). A bounded wait that expires sets kStatusTimeout in *status.
bool tc_gemm_supported(const GemmDesc& g, const EpiDesc& e);
// wait_ns: limit of the pipeline's bounded waits (0: the default 2 s;
// kWaitLimitOff: give up at once, the failure-injection path of the debug GEMM).
constexpr uint64_t kWaitLimitOff = ~0ull;
cudaError_t launch_gemm_tc(cudaStream_t st, const GemmDesc& g, const EpiDesc& e, int sm_count,
                           uint32_t* status, bool pair, uint64_t wait_ns = 0);

// Transpose of a row-major bf16 matrix (rows x cols) into dst (cols x rows,
// row stride ld_dst >= rows; columns [rows, ld_dst) of dst are zeroed).
cudaError_t launch_transpose_bf16(cudaStream_t st, const __nv_bfloat16* src, int64_t rows,
                                  int64_t cols, __nv_bfloat16* dst, int64_t ld_dst);
// H (n bf16 values) as fp16 for the G_W GEMM with the fp16 g operand, in
// two launches: the largest magnitude into *absmax (as float bits; zero it
// first), then dst = fp16(x * 2^-s) with s putting that magnitude in
// [2^14, 2^15), and *epi_scale = 2^s / g_scale for the GEMM epilogue.
cudaError_t launch_absmax_bf16(cudaStream_t st, const __nv_bfloat16* x, int64_t n,
                               uint32_t* absmax);
cudaError_t launch_to_f16_scaled(cudaStream_t st, const __nv_bfloat16* x, int64_t n,
                                 const uint32_t* absmax, float g_scale, __half* dst,
                                 float* epi_scale);
// dst row q = src row (q * mul) mod rows (rows x cols bf16).
cudaError_t launch_permute_rows_bf16(cudaStream_t st, const __nv_bfloat16* src, int64_t rows,
                                     int64_t cols, int64_t mul, __nv_bfloat16* dst);

// MLP helpers.
cudaError_t launch_mlp_delta_a(cudaStream_t st, const dust_params& p, const float* u,
                               int64_t t0, int64_t nt, __nv_bfloat16* da, bool round_bf16,
                               float* da_f32);
cudaError_t launch_reward_gemm_simt(cudaStream_t st, const GemmDesc& g, const float* P,
                                    const int32_t* y, int64_t t0, int32_t K, float* part,
                                    float* dzy);
cudaError_t launch_reward_combine_rows(cudaStream_t st, const float* part, int nparts,
                                       const float* dzy, int64_t rows, int64_t row0, int32_t K,
                                       float* r);
// The perturbed head GEMM contracts only the hi plane of dh = [hi | lo]
// (rows x 2d bf16); this adds the first-order effect of the lo plane to each
// reward: r[t0 K + row] += lo_row . u_t, t = t0 + row / K, with
// u_t = W_head[y_t] - (P W_head)_t (Ut, T x d fp32; P the clean softmax).
// Where dh itself came from the hi plane of da = [hi | lo] (rows x 2 d_ff
// bf16, non-null), it also adds da_lo_row . Wv_t, Wv = u W_down (T x d_ff fp32).
cudaError_t launch_mlp_reward_corr(cudaStream_t st, const __nv_bfloat16* dh, int64_t d,
                                   const float* Ut, const __nv_bfloat16* da, int64_t dff,
                                   const float* Wv, int64_t t0, int32_t K, int64_t rows, float* r);
// U := W_head[y_t] - U row by row (T x d fp32, in place), and bf16(U) into Ub
// (may be null). Targets outside [0, V) take row 0.
cudaError_t launch_head_ut(cudaStream_t st, const __nv_bfloat16* W_head, int64_t V,
                           const int32_t* y, float* U, int64_t T, int64_t d, __nv_bfloat16* Ub,
                           int sm_count);
// out[i] = bf16(x[i]) (round to nearest even), n elements.
cudaError_t launch_f32_to_bf16(cudaStream_t st, const float* x, int64_t n, __nv_bfloat16* out,
                               int sm_count);
// g of the up-projection (width d_ff; gop as bf16 hi/lo planes for bf16 calls)
// or, with down, of the down-projection (width d; gop fp32).
cudaError_t launch_mlp_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                         void* gop, bool down);
// g over width d with counter tag `tag`, gop as bf16 hi/lo planes (T x d each).
cudaError_t launch_noise_g_planes(cudaStream_t st, const dust_params& p, const float* r,
                                  float* g_out, __nv_bfloat16* gop, int tag);
// The same with gop fp32 (T x d).
cudaError_t launch_noise_g_f32(cudaStream_t st, const dust_params& p, const float* r,
                              float* g_out, float* gop, int tag);
// Noise on a width-d output: sigma eps as bf16 hi/lo planes (rows nt K x 2d),
// counter tag `tag` (down projection: 3; attention output projection: 4).
cudaError_t launch_mlp_noise_split(cudaStream_t st, const dust_params& p, int64_t t0, int64_t nt,
                                   __nv_bfloat16* dh, int tag);
// da = GELU(u + du) - GELU(u) for rows (token, draw) of du (fp32, rows x d_ff),
// as bf16 hi/lo planes (rows x 2 d_ff).
cudaError_t launch_gelu_delta_rows(cudaStream_t st, const dust_params& p, const float* u,
                                   const float* du, int64_t t0, int64_t nt, __nv_bfloat16* da);
// a = GELU(u) (fp64, rounded to fp32), n elements.
cudaError_t launch_gelu_f32(cudaStream_t st, const float* u, int64_t n, float* a, int sm_count);
// Attention internals (k_attn.cu): the clean causal attention per (token,
// head) -> O, LSE, gbar = <o, e>; the rewards of noise on the query (which 0)
// or key (1) of every token per head -> part ((T H) x K), summed over heads
// into r (T x K); for the value (2), w = A^T E per head -> W (T x D), then
// the rewards straight into r.
// kcoef: the clean pass also writes the key-noise coefficient rows
size_t attn_fwd_smem(int L, int head_dim, bool kcoef = false);
size_t attn_colsum_smem(int head_dim);
size_t attn_draws_smem(int L, int head_dim);
size_t attn_tc_smem(int L, int head_dim);  // the tensor-core query/key draws (d_h 64, 128)
cudaError_t launch_attn_fwd(cudaStream_t st, int64_t T, int L, int H, int head_dim,
                            const float* Q, const float* Kc, const float* Vc, const float* E,
                            float* O, float* lse, float* gbar, float2* qcoef, float2* kcoef);
cudaError_t launch_attn_draws(cudaStream_t st, const dust_params& p, int which, int L, int H,
                              int head_dim, const float* Q, const float* Kc, const float* Vc,
                              const float* E, const float* O, const float* lse,
                              const float* gbar, float* part, float* W, float* r, bool use_tc,
                              uint8_t* tc_rows, float2* coef, bool coef_done, uint32_t* status);
// bytes of the converted row tiles and of the coefficient rows the
// tensor-core draws read
size_t attn_tc_rows_bytes(int64_t T, int L, int H, int head_dim);
size_t attn_coef_bytes(int64_t T, int L, int H);
cudaError_t launch_attn_combine(cudaStream_t st, const float* part, int64_t T, int H, int K,
                                float* r);

}  // namespace dust
