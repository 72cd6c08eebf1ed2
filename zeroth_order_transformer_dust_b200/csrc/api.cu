// C ABI of the estimator: validation, scratch management and the order of
// the kernel stages. Every numerical step runs in the kernels this file
// launches; nothing here computes on the host beyond index bookkeeping.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "internal.cuh"
#include "noise.cuh"

using namespace dust;

namespace dust {
int64_t default_stride(int64_t V) {
  int64_t a = (int64_t)std::ceil((double)V * ((std::sqrt(5.0) - 1.0) / 2.0));
  if (a < 1) a = 1;
  while (gcd64(a, V) != 1) ++a;
  return a;
}

GopFormat head_gop_format(const dust_params& p) {
  if (p.dtype != DUST_BF16) return GopFormat{kGopF32, 1.0f};
  // Every g entry is bounded by the noise: |r| <= 11.54 sigma and
  // |sigma eps| <= 5.77 sigma (the largest Box-Muller radius of a 24-bit
  // uniform) give |g| <= 66.6 times the entry's inverse-inclusion scale
  // (V/S off the target for subset draws, at most that on it; 1 for the
  // full vocabulary). With 70 for 66.6, g 2^e stays below the fp16 maximum.
  const double scale = p.S > 0 ? (double)p.V / (double)p.S : 1.0;
  const int e = (int)std::floor(std::log2(65504.0 / (70.0 * scale)));
  return GopFormat{kGopF16, std::ldexp(1.0f, e)};
}

size_t gop_format_bytes(GopFormat f, int64_t T, int64_t width) {
  const size_t n = (size_t)T * (size_t)width;
  return f.kind == kGopF32 ? n * 4 : (f.kind == kGopBf16Planes ? n * 4 : n * 2);
}
}  // namespace dust

namespace {

dust_status fail(dust_ctx* ctx, dust_status s, const char* fmt, ...) {
  if (ctx) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    ctx->last_error = buf;
  }
  return s;
}

#define DUST_CU(call)                                                                   \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(ctx, DUST_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define DUST_TRY(expr)            \
  do {                            \
    dust_status s_ = (expr);      \
    if (s_ != DUST_OK) return s_; \
  } while (0)

dust_status check_params(const dust_params* p, int variant, char* msg, int msg_len) {
  auto bad = [&](const char* why) {
    if (msg && msg_len > 0) snprintf(msg, (size_t)msg_len, "%s", why);
    return DUST_ERR_ARG;
  };
  if (!p) return bad("params is NULL");
  if (variant != DUST_VARIANT_HEAD && variant != DUST_VARIANT_MLP && variant != DUST_VARIANT_ATTN)
    return bad("unknown variant");
  const bool attn = variant == DUST_VARIANT_ATTN;
  if (p->T < 1) return bad("T must be >= 1");
  if (p->d < 1) return bad("d must be >= 1");
  if (!attn && p->V < 1) return bad("V must be >= 1");
  if (!attn && p->V > 0x7fffffffLL) return bad("V must fit int32 targets");
  if (p->K < 1) return bad("K must be >= 1");
  if (!std::isfinite(p->sigma) || p->sigma < 0.0f) return bad("sigma must be finite and >= 0");
  if (p->dtype != DUST_F32 && p->dtype != DUST_BF16) return bad("dtype must be DUST_F32 or DUST_BF16");
  if (p->token_offset < 0 || p->token_offset + p->T > (1LL << 32))
    return bad("token_offset + T must lie in [0, 2^32]");
  if (p->draw_offset < 0 || p->draw_offset + (int64_t)p->K > (1LL << 32))
    return bad("draw_offset + K must lie in [0, 2^32]");
  if (p->stream_id >= (1u << 24)) return bad("stream_id must be < 2^24");
  if (!attn && p->T > (1LL << 40) / p->V) return bad("T * V too large");
  if (p->T > (1LL << 40) / p->K) return bad("T * K too large");
  if (variant == DUST_VARIANT_HEAD) {
    if (p->S > p->V) return bad("S must be <= V");
    if (p->S > 0 && p->subset_a != 0) {
      if (p->subset_a < 1) return bad("subset_a must be >= 1");
      if (gcd64(p->subset_a, p->V) != 1) return bad("subset_a must be coprime to V");
    }
  } else if (attn) {
    if (p->S > 0) return bad("the attention variant perturbs every channel: S must be <= 0");
  } else {
    if (p->d_ff < 1) return bad("d_ff must be >= 1");
    if (p->S > 0) return bad("the MLP variant perturbs all d_ff channels: S must be <= 0");
    if (p->dtype != DUST_BF16) return bad("the MLP variant takes bf16 inputs");
    if (p->T > (1LL << 40) / p->d_ff) return bad("T * d_ff too large");
  }
  if (msg && msg_len > 0) msg[0] = 0;
  return DUST_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

dust_status ensure(dust_ctx* ctx, Buf& b, size_t bytes) {
  if (bytes == 0 || b.bytes >= bytes) return DUST_OK;
  if (b.p) {
    cudaStreamSynchronize(ctx->stream);
    cudaFree(b.p);
    b.p = nullptr;
    b.bytes = 0;
  }
  const size_t gran = 2u << 20;
  const size_t nb = (bytes + gran - 1) / gran * gran;
  if (cudaMalloc(&b.p, nb) != cudaSuccess) {
    cudaGetLastError();
    return fail(ctx, DUST_ERR_OOM, "cudaMalloc of %zu bytes failed", nb);
  }
  b.bytes = nb;
  return DUST_OK;
}

dust_status finish(dust_ctx* ctx, uint32_t flags) {
  DUST_CU(cudaGetLastError());
  if (flags & DUST_FLAG_ASYNC) return DUST_OK;
  return dust_check(ctx);
}

// path: 0 automatic, 1 CUDA cores, 2 tensor cores one CTA per tile, 3 tensor
// cores with CTA pairs, 4 as 2 with the pipeline waits' limit at zero (an
// injected timeout).
dust_status run_gemm(dust_ctx* ctx, const GemmDesc& g, const EpiDesc& e, int path = 0) {
  const bool tc = path != 1 && (path >= 2 || ctx->tc_enabled) && tc_gemm_supported(g, e);
  if (path >= 2 && !tc) return fail(ctx, DUST_ERR_UNSUPPORTED, "shape not taken by the tensor-core GEMM");
  ctx->launches += 1;
  if (tc) {
    const bool pair = path == 3 || (path == 0 && ctx->tc_pair && g.M >= 256);
    DUST_CU(launch_gemm_tc(ctx->stream, g, e, ctx->sm_count, ctx->d_status, pair,
                           path == 4 ? kWaitLimitOff : 0));
  } else {
    DUST_CU(launch_gemm_simt(ctx->stream, g, e));
  }
  return DUST_OK;
}

size_t elem_size(int dtype) { return dtype == DUST_BF16 ? 2 : 4; }

// Bytes of the g GEMM operand: fp32, or bf16 hi and lo planes.
size_t gop_bytes(int dtype, int64_t T, int64_t width) {
  return dtype == DUST_BF16 ? (size_t)2 * T * width * 2 : (size_t)T * width * 4;
}

// out (width x N, fp32) = sum_t g_t x_t^T, row w written at (w * row_mul) mod width
// when row_mul != 0. gop holds g (T x width) as fp32 or as bf16 hi/lo planes;
// X is T x N in p.dtype. The bf16 path contracts over 2T (both planes against
// a duplicated X) on tensor cores, reading both operands MN-major as they are
// stored; when their rows are not 16-byte multiples (width or N not a
// multiple of 8) it transposes them to K-major first.
dust_status weight_grad(dust_ctx* ctx, const dust_params& p, const void* gop, int64_t width,
                        const void* X, int64_t N, float* out, int64_t row_mul) {
  const int64_t T = p.T;
  EpiDesc e{};
  e.kind = kEpiF32; e.C = out; e.ldc = N; e.c_row_mul = row_mul;
  if (p.dtype != DUST_BF16) {
    GemmDesc g{};
    g.M = width; g.N = N; g.K = T; g.A = gop; g.lda = width; g.a_kmajor = false;
    g.B = X; g.ldb = N; g.b_kmajor = false; g.dtype = DUST_F32;
    return run_gemm(ctx, g, e);
  }
  const int64_t K2 = 2 * T;
  const size_t xb = (size_t)T * N * 2;
  DUST_TRY(ensure(ctx, ctx->xdup, 2 * xb));
  DUST_CU(cudaMemcpyAsync(ctx->xdup.p, X, xb, cudaMemcpyDeviceToDevice, ctx->stream));
  DUST_CU(cudaMemcpyAsync((char*)ctx->xdup.p + xb, X, xb, cudaMemcpyDeviceToDevice, ctx->stream));
  GemmDesc s{};
  s.M = width; s.N = N; s.K = K2; s.A = gop; s.lda = width; s.a_kmajor = false;
  s.B = ctx->xdup.p; s.ldb = N; s.b_kmajor = false; s.dtype = DUST_BF16;
  if (!ctx->tc_enabled || tc_gemm_supported(s, e)) return run_gemm(ctx, s, e);
  const int64_t ld = (K2 + 7) / 8 * 8;
  DUST_TRY(ensure(ctx, ctx->gT, (size_t)width * ld * 2));
  DUST_TRY(ensure(ctx, ctx->hT, (size_t)N * ld * 2));
  GemmDesc g{};
  g.M = width; g.N = N; g.K = K2; g.A = ctx->gT.p; g.lda = ld; g.a_kmajor = true;
  g.B = ctx->hT.p; g.ldb = ld; g.b_kmajor = true; g.dtype = DUST_BF16;
  if (ctx->tc_enabled && tc_gemm_supported(g, e)) {
    DUST_CU(launch_transpose_bf16(ctx->stream, (const __nv_bfloat16*)gop, K2, width,
                                  (__nv_bfloat16*)ctx->gT.p, ld));
    DUST_CU(launch_transpose_bf16(ctx->stream, (const __nv_bfloat16*)ctx->xdup.p, K2, N,
                                  (__nv_bfloat16*)ctx->hT.p, ld));
    ctx->launches += 2;
    return run_gemm(ctx, g, e);
  }
  return run_gemm(ctx, s, e);
}

// out (width x N, fp32) = sum_t g_t x_t^T from the fp16 g operand (g * gscale,
// T x width) and bf16 X (T x N): X is converted to fp16 with a power-of-two
// scale from its largest magnitude (on the device), and the GEMM (K = T, both
// operands MN-major as stored) multiplies its sums by the two scales'
// inverse. Rows that are not 16-byte multiples are transposed to K-major
// first; without tensor cores the CUDA-core GEMM reads the fp16 operands.
dust_status weight_grad_f16(dust_ctx* ctx, const dust_params& p, const void* gop, float gscale,
                            int64_t width, const void* X, int64_t N, float* out,
                            int64_t row_mul) {
  const int64_t T = p.T;
  DUST_TRY(ensure(ctx, ctx->xdup, (size_t)T * N * 2));
  DUST_TRY(ensure(ctx, ctx->hsc, 16));
  uint32_t* absmax = (uint32_t*)ctx->hsc.p;
  float* escale = (float*)ctx->hsc.p + 1;
  DUST_CU(cudaMemsetAsync(absmax, 0, sizeof(uint32_t), ctx->stream));
  DUST_CU(launch_absmax_bf16(ctx->stream, (const __nv_bfloat16*)X, T * N, absmax));
  DUST_CU(launch_to_f16_scaled(ctx->stream, (const __nv_bfloat16*)X, T * N, absmax, gscale,
                               (__half*)ctx->xdup.p, escale));
  ctx->launches += 2;
  EpiDesc e{};
  e.kind = kEpiF32; e.C = out; e.ldc = N; e.c_row_mul = row_mul; e.scale = escale;
  GemmDesc s{};
  s.M = width; s.N = N; s.K = T; s.A = gop; s.lda = width; s.a_kmajor = false;
  s.B = ctx->xdup.p; s.ldb = N; s.b_kmajor = false; s.dtype = DUST_BF16; s.f16 = true;
  if (!ctx->tc_enabled || tc_gemm_supported(s, e)) return run_gemm(ctx, s, e);
  const int64_t ld = (T + 7) / 8 * 8;
  DUST_TRY(ensure(ctx, ctx->gT, (size_t)width * ld * 2));
  DUST_TRY(ensure(ctx, ctx->hT, (size_t)N * ld * 2));
  GemmDesc g{};
  g.M = width; g.N = N; g.K = T; g.A = ctx->gT.p; g.lda = ld; g.a_kmajor = true;
  g.B = ctx->hT.p; g.ldb = ld; g.b_kmajor = true; g.dtype = DUST_BF16; g.f16 = true;
  if (tc_gemm_supported(g, e)) {
    // the transposes move 2-byte words, whatever their type
    DUST_CU(launch_transpose_bf16(ctx->stream, (const __nv_bfloat16*)gop, T, width,
                                  (__nv_bfloat16*)ctx->gT.p, ld));
    DUST_CU(launch_transpose_bf16(ctx->stream, (const __nv_bfloat16*)ctx->xdup.p, T, N,
                                  (__nv_bfloat16*)ctx->hT.p, ld));
    ctx->launches += 2;
    return run_gemm(ctx, g, e);
  }
  return run_gemm(ctx, s, e);
}

// The full-vocabulary draws split over two streams (full_split_plan): the one-pass
// kernel over tokens [0, T - T2) at the higher priority, so that its clusters are
// placed first, and the two passes over the last T2 tokens at the lower, their
// CTAs kept off the one-pass SMs. Both streams fork from the call's stream after
// the log-sum-exp and join it before the G_W GEMM; the join is recorded even
// when a launch fails.
dust_status full_split_draws(dust_ctx* ctx, const dust_params& p, const FullOnePlan& one,
                             const FullSide& side, int64_t T2, const float* Z,
                             const int32_t* targets, float* rewards_out, float* g_out,
                             GopFormat gf) {
  // made at first use; what a failed attempt left unmade is made by the next
  if (!ctx->side_hi || !ctx->side_lo || !ctx->fork_ev || !ctx->join_hi || !ctx->join_lo) {
    int least = 0, greatest = 0;
    DUST_CU(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    if (!ctx->side_hi)
      DUST_CU(cudaStreamCreateWithPriority(&ctx->side_hi, cudaStreamNonBlocking, greatest));
    if (!ctx->side_lo)
      DUST_CU(cudaStreamCreateWithPriority(&ctx->side_lo, cudaStreamNonBlocking, least));
    for (cudaEvent_t* ev : {&ctx->fork_ev, &ctx->join_hi, &ctx->join_lo})
      if (!*ev) DUST_CU(cudaEventCreateWithFlags(ev, cudaEventDisableTiming));
  }
  const int64_t T1 = p.T - T2;
  dust_params p1 = p, p2 = p;
  p1.T = T1;
  p2.T = T2;
  p2.token_offset = p.token_offset + T1;
  float* r2 = rewards_out ? rewards_out + T1 * p.K : nullptr;
  if (!r2) {
    DUST_TRY(ensure(ctx, ctx->rew, (size_t)T2 * p.K * 4));
    r2 = (float*)ctx->rew.p;
  }
  DUST_TRY(ensure(ctx, ctx->part, (size_t)T2 * full_vocab_nslab(p.V) * p.K * 4));
  DUST_TRY(ensure(ctx, ctx->dzy, full_vocab_xy_bytes(T2, p.K)));
  const float* lse = (const float*)ctx->lse.p;
  const size_t esz = gf.kind == kGopF32 ? 4 : 2;
  void* gop2 = (char*)ctx->gop.p + (size_t)T1 * p.V * esz;
  const cudaStream_t st = ctx->stream;
  DUST_CU(cudaEventRecord(ctx->fork_ev, st));
  DUST_CU(cudaStreamWaitEvent(ctx->side_hi, ctx->fork_ev, 0));
  DUST_CU(cudaStreamWaitEvent(ctx->side_lo, ctx->fork_ev, 0));
  cudaError_t e = launch_full_one(ctx->side_hi, p1, one, Z, lse, targets, rewards_out, g_out,
                                  ctx->gop.p, gf, ctx->d_status);
  if (e == cudaSuccess)
    e = launch_full_reward_partial(ctx->side_lo, p2, Z + T1 * p.V, lse + T1, targets + T1,
                                   (float*)ctx->part.p, (float*)ctx->dzy.p, &side);
  if (e == cudaSuccess)
    e = launch_full_reward_combine(ctx->side_lo, p2, (float*)ctx->part.p, (float*)ctx->dzy.p, r2);
  if (e == cudaSuccess)
    e = launch_full_g(ctx->side_lo, p2, r2, g_out ? g_out + T1 * p.V : nullptr, gop2, gf, &side);
  DUST_CU(cudaEventRecord(ctx->join_hi, ctx->side_hi));
  DUST_CU(cudaEventRecord(ctx->join_lo, ctx->side_lo));
  DUST_CU(cudaStreamWaitEvent(st, ctx->join_hi, 0));
  DUST_CU(cudaStreamWaitEvent(st, ctx->join_lo, 0));
  DUST_CU(e);
  ctx->launches += 4;
  return DUST_OK;
}

// Stage marks: mark(ctx, nullptr) opens a call, mark(ctx, "name") closes the
// stage that ran since the previous mark.
void mark(dust_ctx* ctx, const char* name) {
  if (!ctx->timing) return;
  if (!name) ctx->nmarks = 0;
  if (ctx->nmarks >= dust_ctx::kMaxMarks) return;
  cudaEventRecord(ctx->ev[ctx->nmarks], ctx->stream);
  ctx->mark_name[ctx->nmarks] = name;
  ctx->nmarks++;
}

}  // namespace

extern "C" {

const char* dust_status_string(dust_status s) {
  switch (s) {
    case DUST_OK: return "DUST_OK";
    case DUST_ERR_ARG: return "DUST_ERR_ARG";
    case DUST_ERR_CUDA: return "DUST_ERR_CUDA";
    case DUST_ERR_OOM: return "DUST_ERR_OOM";
    case DUST_ERR_BOUNDS: return "DUST_ERR_BOUNDS";
    case DUST_ERR_TIMEOUT: return "DUST_ERR_TIMEOUT";
    case DUST_ERR_UNSUPPORTED: return "DUST_ERR_UNSUPPORTED";
  }
  return "DUST_ERR_UNKNOWN";
}

dust_status dust_validate(const dust_params* p, int variant, char* msg, int msg_len) {
  return check_params(p, variant, msg, msg_len);
}

int64_t dust_subset_stride(const dust_params* p) {
  if (check_params(p, DUST_VARIANT_HEAD, nullptr, 0) != DUST_OK || p->S <= 0) return 0;
  return subset_stride_of(*p);
}

dust_status dust_create(dust_ctx** out, int device, void* cuda_stream) {
  if (!out) return DUST_ERR_ARG;
  *out = nullptr;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return DUST_ERR_CUDA;
  }
  dust_ctx* ctx = new dust_ctx();
  ctx->device = device;
  ctx->stream = (cudaStream_t)cuda_stream;
  const char* no_tc = getenv("DUST_DISABLE_TC");
  ctx->tc_enabled = !(no_tc && no_tc[0] && no_tc[0] != '0');
  const char* pair = getenv("DUST_TC_PAIR");
  ctx->tc_pair = !(pair && pair[0] == '0');
  const char* sk = getenv("DUST_SUBSET_KERNEL");
  ctx->subset2_enabled = !(sk && sk[0] == '1');
  const char* fk = getenv("DUST_FULL_KERNEL");
  ctx->full_one_enabled = !(fk && fk[0] == '2');
  const char* fs = getenv("DUST_FULL_SPLIT");
  ctx->full_split = !(fs && fs[0] == '0');
  if (cudaSetDevice(device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess ||
      cudaMalloc(&ctx->d_status, sizeof(uint32_t)) != cudaSuccess ||
      cudaMallocHost(&ctx->h_status, sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(ctx->d_status, 0, sizeof(uint32_t)) != cudaSuccess) {
    cudaGetLastError();
    dust_destroy(ctx);
    return DUST_ERR_CUDA;
  }
  *out = ctx;
  return DUST_OK;
}

dust_status dust_set_stream(dust_ctx* ctx, void* cuda_stream) {
  if (!ctx) return DUST_ERR_ARG;
  ctx->stream = (cudaStream_t)cuda_stream;
  return DUST_OK;
}

void dust_destroy(dust_ctx* ctx) {
  if (!ctx) return;
  cudaSetDevice(ctx->device);
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  for (cudaStream_t s : {ctx->side_hi, ctx->side_lo})
    if (s) cudaStreamSynchronize(s);
  Buf* bufs[] = {&ctx->z, &ctx->lse, &ctx->loss, &ctx->gop, &ctx->rew, &ctx->part, &ctx->wperm,
                 &ctx->gT, &ctx->hT, &ctx->xdup, &ctx->dzy, &ctx->mlp_u, &ctx->mlp_a, &ctx->mlp_h,
                 &ctx->mlp_da, &ctx->mlp_dh, &ctx->wd2, &ctx->wh2, &ctx->in_h, &ctx->in_w, &ctx->in_y, &ctx->out_g,
                 &ctx->out_loss, &ctx->out_r, &ctx->out_gv, &ctx->lsep, &ctx->mlp_a32,
                 &ctx->mlp_dn, &ctx->mlp_du, &ctx->wu2, &ctx->attn_o, &ctx->attn_lse,
                 &ctx->attn_gb, &ctx->attn_w, &ctx->attn_tcr, &ctx->attn_coef, &ctx->hsc,
                 &ctx->mlp_pb, &ctx->mlp_uw, &ctx->mlp_ub, &ctx->mlp_wv, &ctx->mlp_wt};
  for (Buf* b : bufs)
    if (b->p) cudaFree(b->p);
  for (int i = 0; i < dust_ctx::kMaxMarks; ++i)
    if (ctx->ev[i]) cudaEventDestroy(ctx->ev[i]);
  for (cudaStream_t s : {ctx->side_hi, ctx->side_lo})
    if (s) cudaStreamDestroy(s);
  for (cudaEvent_t e : {ctx->fork_ev, ctx->join_hi, ctx->join_lo})
    if (e) cudaEventDestroy(e);
  if (ctx->d_status) cudaFree(ctx->d_status);
  if (ctx->h_status) cudaFreeHost(ctx->h_status);
  cudaGetLastError();
  delete ctx;
}

const char* dust_last_error(const dust_ctx* ctx) {
  return ctx ? ctx->last_error.c_str() : "no context";
}

dust_status dust_check(dust_ctx* ctx) {
  if (!ctx) return DUST_ERR_ARG;
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(cudaMemcpyAsync(ctx->h_status, ctx->d_status, sizeof(uint32_t), cudaMemcpyDeviceToHost,
                          ctx->stream));
  DUST_CU(cudaStreamSynchronize(ctx->stream));
  const uint32_t st = *ctx->h_status;
  if (st) DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), ctx->stream));
  if (st & kStatusBadTarget) return fail(ctx, DUST_ERR_BOUNDS, "a target lies outside [0, V)");
  if (st & kStatusTimeout) return fail(ctx, DUST_ERR_TIMEOUT, "a bounded device wait expired");
  if (st & kStatusRange)
    return fail(ctx, DUST_ERR_UNSUPPORTED,
                "a query or key value lies outside the fp16 range of the tensor-core attention "
                "path (|x| < 32768); DUST_ATTN_TC=0 selects the CUDA-core path");
  return DUST_OK;
}

dust_status dust_head_grad(dust_ctx* ctx, const dust_params* pp, const void* H, const void* W,
                           const int32_t* targets, float* G_out, float* loss_out,
                           float* rewards_out, float* g_out) {
  if (!ctx) return DUST_ERR_ARG;
  char why[256];
  if (check_params(pp, DUST_VARIANT_HEAD, why, sizeof(why)) != DUST_OK)
    return fail(ctx, DUST_ERR_ARG, "%s", why);
  const dust_params p = *pp;
  if (!H || !W || !targets) return fail(ctx, DUST_ERR_ARG, "H, W and targets must be non-NULL");
  if (!aligned(H, 16) || !aligned(W, 16) || !aligned(targets, 4) || !aligned(G_out, 4) ||
      !aligned(loss_out, 4) || !aligned(rewards_out, 4) || !aligned(g_out, 4))
    return fail(ctx, DUST_ERR_ARG, "H and W must be 16-byte aligned, the other pointers 4-byte");
  DUST_CU(cudaSetDevice(ctx->device));
  const bool subset = p.S > 0;
  const int64_t a = subset ? subset_stride_of(p) : 0;
  const int64_t a_inv = subset ? modinv(a, p.V) : 0;
  const size_t TV = (size_t)p.T * (size_t)p.V;
  DUST_TRY(ensure(ctx, ctx->z, TV * 4));
  DUST_TRY(ensure(ctx, ctx->lse, (size_t)p.T * 4));
  const GopFormat gf = head_gop_format(p);
  DUST_TRY(ensure(ctx, ctx->gop, gop_format_bytes(gf, p.T, p.V)));
  float* loss = loss_out;
  if (!loss) {
    DUST_TRY(ensure(ctx, ctx->loss, (size_t)p.T * 4));
    loss = (float*)ctx->loss.p;
  }
  float* Z = (float*)ctx->z.p;
  const cudaStream_t st = ctx->stream;
  DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), st));
  mark(ctx, nullptr);

  // 1. clean logits z = H W^T (permuted columns for subset draws: the bf16
  //    path gathers the rows of W once so the tensor-core GEMM reads them
  //    contiguously; the CUDA-core path gathers on the fly)
  const void* Wuse = W;
  int64_t bmul = subset ? a : 0;
  if (subset && p.dtype == DUST_BF16) {
    DUST_TRY(ensure(ctx, ctx->wperm, (size_t)p.V * p.d * 2));
    DUST_CU(launch_permute_rows_bf16(st, (const __nv_bfloat16*)W, p.V, p.d, a,
                                     (__nv_bfloat16*)ctx->wperm.p));
    ctx->launches += 1;
    Wuse = ctx->wperm.p;
    bmul = 0;
  }
  GemmDesc g{};
  g.M = p.T; g.N = p.V; g.K = p.d;
  g.A = H; g.lda = p.d; g.a_kmajor = true;
  g.B = Wuse; g.ldb = p.d; g.b_kmajor = true;
  g.b_row_mul = bmul;
  g.dtype = p.dtype;
  EpiDesc e{};
  e.kind = kEpiF32; e.C = Z; e.ldc = p.V;
  // The draw kernels form p = exp(z - LSE) themselves, except the L2-fed
  // subset kernel, which reads p written in place over z.
  const bool smem_subset =
      subset && ctx->subset2_enabled && subset2_cluster_size(p.V, p.S, ctx->max_smem_optin) > 0;
  const bool need_prob = subset && !smem_subset;
  // On tensor cores the GEMM epilogue also leaves per-tile softmax partials
  // of every row (the per-token max / log-sum-exp cache), so z is not re-read.
  const bool fused = !need_prob && ctx->tc_enabled && tc_gemm_supported(g, e);
  const int ntiles = tc_partials_per_row(p.V);
  if (fused) {
    DUST_TRY(ensure(ctx, ctx->lsep, (size_t)p.T * ntiles * sizeof(float2)));
    e.kind = kEpiF32Lse;
    e.lsep = (float2*)ctx->lsep.p;
  }
  DUST_TRY(run_gemm(ctx, g, e));
  mark(ctx, "clean_gemm");
  // 2. log-sum-exp and clean loss
  if (fused)
    DUST_CU(launch_lse_combine(st, (const float2*)ctx->lsep.p, ntiles, Z, p.T, p.V, targets,
                               subset ? a_inv : 0, (float*)ctx->lse.p, loss, ctx->d_status));
  else
    DUST_CU(launch_lse_rows(st, Z, p.T, p.V, targets, subset ? a_inv : 0, (float*)ctx->lse.p,
                            loss, need_prob, ctx->d_status));
  ctx->launches += 1;
  mark(ctx, "lse");
  // 3. perturbed losses, rewards, g
  FullOnePlan one;
  if (!subset && ctx->full_one_enabled &&
      full_one_plan(p, ctx->sm_count, ctx->max_smem_optin, &one)) {
    FullSide side;
    const int64_t T2 = ctx->full_split && gf.kind != kGopBf16Planes
                           ? full_split_plan(p, one, ctx->sm_count, &side)
                           : 0;
    if (T2 > 0) {
      DUST_TRY(full_split_draws(ctx, p, one, side, T2, Z, targets, rewards_out, g_out, gf));
    } else {
      DUST_CU(launch_full_one(st, p, one, Z, (const float*)ctx->lse.p, targets, rewards_out,
                              g_out, ctx->gop.p, gf, ctx->d_status));
      ctx->launches += 1;
    }
    mark(ctx, "full_draws");
  } else if (!subset) {
    float* r = rewards_out;
    if (!r) {
      DUST_TRY(ensure(ctx, ctx->rew, (size_t)p.T * p.K * 4));
      r = (float*)ctx->rew.p;
    }
    DUST_TRY(ensure(ctx, ctx->part, (size_t)p.T * full_vocab_nslab(p.V) * p.K * 4));
    DUST_TRY(ensure(ctx, ctx->dzy, full_vocab_xy_bytes(p.T, p.K)));
    DUST_CU(launch_full_reward_partial(st, p, Z, (const float*)ctx->lse.p, targets,
                                       (float*)ctx->part.p, (float*)ctx->dzy.p));
    DUST_CU(launch_full_reward_combine(st, p, (float*)ctx->part.p, (float*)ctx->dzy.p, r));
    ctx->launches += 2;
    mark(ctx, "reward");
    DUST_CU(launch_full_g(st, p, r, g_out, ctx->gop.p, gf));
    ctx->launches += 1;
    mark(ctx, "g");
  } else if (smem_subset) {
    DUST_CU(launch_subset2(st, p, a, a_inv, Z, (const float*)ctx->lse.p, targets, rewards_out,
                           g_out, ctx->gop.p, gf, ctx->max_smem_optin, ctx->sm_count,
                           ctx->d_status));
    ctx->launches += 1;
    mark(ctx, "subset_draws");
  } else {
    float* gacc = nullptr;
    const size_t gb = subset_gacc_bytes(p.T, p.V, ctx->max_smem_optin);
    if (gb) {
      DUST_TRY(ensure(ctx, ctx->part, gb));
      gacc = (float*)ctx->part.p;
    }
    DUST_CU(launch_subset_impl(st, p, a, a_inv, Z, targets, rewards_out, g_out, ctx->gop.p, gf, gacc,
                               ctx->max_smem_optin));
    ctx->launches += 1;
    mark(ctx, "subset_draws");
  }
  // 4. G_W = sum_t g_t h_t^T (rows un-permuted on the store)
  if (G_out) {
    if (gf.kind == kGopF16)
      DUST_TRY(weight_grad_f16(ctx, p, ctx->gop.p, gf.scale, p.V, H, p.d, G_out, subset ? a : 0));
    else
      DUST_TRY(weight_grad(ctx, p, ctx->gop.p, p.V, H, p.d, G_out, subset ? a : 0));
    mark(ctx, "gw_gemm");
  }
  return finish(ctx, p.flags);
}

dust_status dust_head_grad_host(dust_ctx* ctx, const dust_params* pp, const void* H, const void* W,
                                const int32_t* targets, float* G_out, float* loss_out,
                                float* rewards_out, float* g_out) {
  if (!ctx) return DUST_ERR_ARG;
  char why[256];
  if (check_params(pp, DUST_VARIANT_HEAD, why, sizeof(why)) != DUST_OK)
    return fail(ctx, DUST_ERR_ARG, "%s", why);
  if (!H || !W || !targets) return fail(ctx, DUST_ERR_ARG, "H, W and targets must be non-NULL");
  const dust_params p = *pp;
  DUST_CU(cudaSetDevice(ctx->device));
  const size_t es = elem_size(p.dtype);
  const size_t hb = (size_t)p.T * p.d * es, wb = (size_t)p.V * p.d * es, yb = (size_t)p.T * 4;
  DUST_TRY(ensure(ctx, ctx->in_h, hb));
  DUST_TRY(ensure(ctx, ctx->in_w, wb));
  DUST_TRY(ensure(ctx, ctx->in_y, yb));
  if (G_out) DUST_TRY(ensure(ctx, ctx->out_g, (size_t)p.V * p.d * 4));
  if (loss_out) DUST_TRY(ensure(ctx, ctx->out_loss, (size_t)p.T * 4));
  if (rewards_out) DUST_TRY(ensure(ctx, ctx->out_r, (size_t)p.T * p.K * 4));
  if (g_out) DUST_TRY(ensure(ctx, ctx->out_gv, (size_t)p.T * p.V * 4));
  const cudaStream_t st = ctx->stream;
  DUST_CU(cudaMemcpyAsync(ctx->in_h.p, H, hb, cudaMemcpyHostToDevice, st));
  DUST_CU(cudaMemcpyAsync(ctx->in_w.p, W, wb, cudaMemcpyHostToDevice, st));
  DUST_CU(cudaMemcpyAsync(ctx->in_y.p, targets, yb, cudaMemcpyHostToDevice, st));
  dust_params q = p;
  q.flags |= DUST_FLAG_ASYNC;
  DUST_TRY(dust_head_grad(ctx, &q, ctx->in_h.p, ctx->in_w.p, (const int32_t*)ctx->in_y.p,
                          G_out ? (float*)ctx->out_g.p : nullptr,
                          loss_out ? (float*)ctx->out_loss.p : nullptr,
                          rewards_out ? (float*)ctx->out_r.p : nullptr,
                          g_out ? (float*)ctx->out_gv.p : nullptr));
  if (G_out) DUST_CU(cudaMemcpyAsync(G_out, ctx->out_g.p, (size_t)p.V * p.d * 4, cudaMemcpyDeviceToHost, st));
  if (loss_out) DUST_CU(cudaMemcpyAsync(loss_out, ctx->out_loss.p, (size_t)p.T * 4, cudaMemcpyDeviceToHost, st));
  if (rewards_out) DUST_CU(cudaMemcpyAsync(rewards_out, ctx->out_r.p, (size_t)p.T * p.K * 4, cudaMemcpyDeviceToHost, st));
  if (g_out) DUST_CU(cudaMemcpyAsync(g_out, ctx->out_gv.p, (size_t)p.T * p.V * 4, cudaMemcpyDeviceToHost, st));
  if (p.flags & DUST_FLAG_ASYNC) {
    DUST_CU(cudaStreamSynchronize(st));
    return DUST_OK;
  }
  return dust_check(ctx);
}

// The MLP-block layer variants share the clean pass and the reward GEMM; the
// perturbed layer decides the head-input change dh of each draw:
//   kLayerUp:      noise on u = W_up x,    dh = (GELU(u + s e) - GELU(u)) W_down^T
//   kLayerDown:    noise on W_down's output, dh = s e
//   kLayerAttnOut: noise on W_o o, the residual x entering the block:
//                  du = s e W_up^T, dh = s e + (GELU(u + du) - GELU(u)) W_down^T
enum MlpLayer { kLayerUp = 0, kLayerDown = 1, kLayerAttnOut = 2 };

static dust_status mlp_impl(dust_ctx* ctx, const dust_params* pp, int layer, const void* X,
                            const void* O, int64_t d_o, const void* W_up, const void* W_down,
                            const void* W_head, const int32_t* targets, float* G_out,
                            float* loss_out, float* rewards_out, float* g_out) {
  const bool down = layer == kLayerDown, attn = layer == kLayerAttnOut;
  if (!ctx) return DUST_ERR_ARG;
  char why[256];
  if (check_params(pp, DUST_VARIANT_MLP, why, sizeof(why)) != DUST_OK)
    return fail(ctx, DUST_ERR_ARG, "%s", why);
  const dust_params p = *pp;
  if (!X || !W_up || !W_down || !W_head || !targets)
    return fail(ctx, DUST_ERR_ARG, "X, W_up, W_down, W_head and targets must be non-NULL");
  if (attn && (!O || d_o < 1 || (d_o & 7) || !aligned(O, 16)))
    return fail(ctx, DUST_ERR_ARG, "O must be non-NULL and 16-byte aligned, d_o >= 1 a multiple of 8");
  if (!aligned(X, 16) || !aligned(W_up, 16) || !aligned(W_down, 16) || !aligned(W_head, 16) ||
      !aligned(targets, 4) || !aligned(G_out, 4) || !aligned(loss_out, 4) ||
      !aligned(rewards_out, 4) || !aligned(g_out, 4))
    return fail(ctx, DUST_ERR_ARG, "weights and X must be 16-byte aligned, the rest 4-byte");
  DUST_CU(cudaSetDevice(ctx->device));
  const cudaStream_t st = ctx->stream;
  const int64_t T = p.T, d = p.d, dff = p.d_ff, V = p.V, K = p.K;
  DUST_TRY(ensure(ctx, ctx->mlp_u, (size_t)T * dff * 4));
  DUST_TRY(ensure(ctx, ctx->mlp_a, (size_t)T * 2 * dff * 2));
  DUST_TRY(ensure(ctx, ctx->mlp_h, (size_t)T * 2 * d * 2));
  DUST_TRY(ensure(ctx, ctx->z, (size_t)T * V * 4));
  DUST_TRY(ensure(ctx, ctx->lse, (size_t)T * 4));
  DUST_TRY(ensure(ctx, ctx->gop, down ? (size_t)T * d * 4
                                       : gop_bytes(DUST_BF16, T, attn ? d : dff)));
  float* loss = loss_out;
  if (!loss) {
    DUST_TRY(ensure(ctx, ctx->loss, (size_t)T * 4));
    loss = (float*)ctx->loss.p;
  }
  float* r = rewards_out;
  if (!r) {
    DUST_TRY(ensure(ctx, ctx->rew, (size_t)T * K * 4));
    r = (float*)ctx->rew.p;
  }
  float* u = (float*)ctx->mlp_u.p;
  __nv_bfloat16* abf = (__nv_bfloat16*)ctx->mlp_a.p;
  __nv_bfloat16* hbf = (__nv_bfloat16*)ctx->mlp_h.p;
  float* Z = (float*)ctx->z.p;
  DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), st));
  mark(ctx, nullptr);

  // clean pass, activations at full precision as bf16 hi/lo planes:
  //   u = x W_up^T (fp32); a = GELU(u) (fp64) -> [a_hi | a_lo] (T x 2 d_ff);
  //   h = x + a W_down^T -> [h_hi | h_lo] (T x 2d); z = h W_head^T.
  // The planes are contracted against weights duplicated along K.
  DUST_TRY(ensure(ctx, ctx->wd2, (size_t)d * 2 * dff * 2));
  DUST_TRY(ensure(ctx, ctx->wh2, (size_t)V * 2 * d * 2));
  for (int half = 0; half < 2; ++half) {
    DUST_CU(cudaMemcpy2DAsync((char*)ctx->wd2.p + (size_t)half * dff * 2, (size_t)2 * dff * 2,
                              W_down, (size_t)dff * 2, (size_t)dff * 2, (size_t)d,
                              cudaMemcpyDeviceToDevice, st));
    DUST_CU(cudaMemcpy2DAsync((char*)ctx->wh2.p + (size_t)half * d * 2, (size_t)2 * d * 2, W_head,
                              (size_t)d * 2, (size_t)d * 2, (size_t)V, cudaMemcpyDeviceToDevice, st));
  }
  {
    GemmDesc g{};
    g.M = T; g.N = dff; g.K = d; g.A = X; g.lda = d; g.a_kmajor = true;
    g.B = W_up; g.ldb = d; g.b_kmajor = true; g.dtype = DUST_BF16;
    EpiDesc e{};
    e.kind = kEpiGeluSplit; e.C = u; e.ldc = dff; e.Cb = abf; e.ldcb = 2 * dff; e.split = dff;
    DUST_TRY(run_gemm(ctx, g, e));
  }
  {
    GemmDesc g{};
    g.M = T; g.N = d; g.K = 2 * dff; g.A = abf; g.lda = 2 * dff; g.a_kmajor = true;
    g.B = ctx->wd2.p; g.ldb = 2 * dff; g.b_kmajor = true; g.dtype = DUST_BF16;
    EpiDesc e{};
    e.kind = kEpiResidSplit; e.Cb = hbf; e.ldcb = 2 * d; e.split = d; e.resid = X; e.ldr = d;
    DUST_TRY(run_gemm(ctx, g, e));
  }
  {
    GemmDesc g{};
    g.M = T; g.N = V; g.K = 2 * d; g.A = hbf; g.lda = 2 * d; g.a_kmajor = true;
    g.B = ctx->wh2.p; g.ldb = 2 * d; g.b_kmajor = true; g.dtype = DUST_BF16;
    EpiDesc e{};
    e.kind = kEpiF32; e.C = Z; e.ldc = V;
    DUST_TRY(run_gemm(ctx, g, e));
  }
  mark(ctx, "clean_gemms");
  DUST_CU(launch_lse_rows(st, Z, T, V, targets, 0, (float*)ctx->lse.p, loss, true, ctx->d_status));
  ctx->launches += 1;
  mark(ctx, "lse");
  // U = P W_head (T x d, fp32) from the softmax P (now in Z) rounded to bf16:
  // the perturbed rewards take the head GEMM on the hi plane of dh only and add
  // the lo plane's first-order effect, lo . (W_head[y_t] - U_t), per row.
  // (The dropped terms are of second order in the lo plane, in Delta z and in
  // P's rounding: about 6e-8 on the rewards and 3e-6 relative on g in the
  // oracle's arithmetic on the mlp_bf16 shapes, against 2e-5 and 1e-4.)
  // The dropped terms grow as sigma^2 (the oracle's rewards: 2.8e-6 at sigma =
  // 0.05, 9e-6 at 0.1, 4e-5 at 0.2 on small shapes), so above sigma = 0.05 the
  // GEMMs contract both planes (K = 2d and 2 d_ff, against the weights
  // duplicated along K) and no correction is made.
  const bool one_plane = p.sigma <= 0.05f;
  float* Uw = nullptr;
  float* Wv = nullptr;
  if (one_plane) {
    // (both GEMMs K-major: W_head and W_down transposed once per call)
    const int64_t ldv = (V + 7) / 8 * 8, ldd = (d + 7) / 8 * 8;
    DUST_TRY(ensure(ctx, ctx->mlp_pb, (size_t)T * V * 2));
    DUST_TRY(ensure(ctx, ctx->mlp_uw, (size_t)T * d * 4));
    DUST_TRY(ensure(ctx, ctx->mlp_wt, (size_t)std::max(d * ldv, dff * ldd) * 2));
    Uw = (float*)ctx->mlp_uw.p;
    DUST_CU(launch_f32_to_bf16(st, Z, T * V, (__nv_bfloat16*)ctx->mlp_pb.p, ctx->sm_count));
    DUST_CU(launch_transpose_bf16(st, (const __nv_bfloat16*)W_head, V, d,
                                  (__nv_bfloat16*)ctx->mlp_wt.p, ldv));
    ctx->launches += 2;
    {
      GemmDesc g{};
      g.M = T; g.N = d; g.K = V; g.A = ctx->mlp_pb.p; g.lda = V; g.a_kmajor = true;
      g.B = ctx->mlp_wt.p; g.ldb = ldv; g.b_kmajor = true; g.dtype = DUST_BF16;
      EpiDesc e{};
      e.kind = kEpiF32; e.C = Uw; e.ldc = d;
      DUST_TRY(run_gemm(ctx, g, e));
    }
    // u_t = W_head[y_t] - U_t in place of U (and in bf16 where Wv needs it).
    // Where dh = da W_down^T (up-projection, attention output projection), that
    // GEMM too contracts only the hi plane of da; the lo plane moves a reward by
    // da_lo . Wv_t to first order, Wv = u W_down (T x d_ff, from u in bf16).
    // With both corrections the oracle's rewards move by 1.1e-7 and g by 4.9e-6
    // relative on the mlp_bf16 shapes.
    if (!down) DUST_TRY(ensure(ctx, ctx->mlp_ub, (size_t)T * d * 2));
    DUST_CU(launch_head_ut(st, (const __nv_bfloat16*)W_head, V, targets, Uw, T, d,
                           down ? nullptr : (__nv_bfloat16*)ctx->mlp_ub.p, ctx->sm_count));
    ctx->launches += 1;
    if (!down) {
      DUST_TRY(ensure(ctx, ctx->mlp_wv, (size_t)T * dff * 4));
      Wv = (float*)ctx->mlp_wv.p;
      DUST_CU(launch_transpose_bf16(st, (const __nv_bfloat16*)W_down, d, dff,
                                    (__nv_bfloat16*)ctx->mlp_wt.p, ldd));
      ctx->launches += 1;
      GemmDesc g{};
      g.M = T; g.N = dff; g.K = d; g.A = ctx->mlp_ub.p; g.lda = d; g.a_kmajor = true;
      g.B = ctx->mlp_wt.p; g.ldb = ldd; g.b_kmajor = true; g.dtype = DUST_BF16;
      EpiDesc e{};
      e.kind = kEpiF32; e.C = Wv; e.ldc = dff;
      DUST_TRY(run_gemm(ctx, g, e));
    }
    mark(ctx, "head_mean");
  }

  // perturbed passes, a chunk of tokens (all K draws each) at a time
  const int64_t max_rows = 131072;
  int64_t tchunk = max_rows / K;
  if (tchunk < 1) tchunk = 1;
  if (tchunk > T) tchunk = T;
  const int64_t rows_cap = tchunk * K;
  // reward partials per row: 128-column tiles on CUDA cores, two per 256-column tile on
  // tensor cores
  const int nparts = std::max((int)((V + 127) / 128), tc_partials_per_row(V));
  if (!down) DUST_TRY(ensure(ctx, ctx->mlp_da, (size_t)rows_cap * 2 * dff * 2));
  if (attn) {
    DUST_TRY(ensure(ctx, ctx->mlp_dn, (size_t)rows_cap * 2 * d * 2));
    DUST_TRY(ensure(ctx, ctx->mlp_du, (size_t)rows_cap * dff * 4));
    DUST_TRY(ensure(ctx, ctx->wu2, (size_t)dff * 2 * d * 2));
    for (int half = 0; half < 2; ++half)
      DUST_CU(cudaMemcpy2DAsync((char*)ctx->wu2.p + (size_t)half * d * 2, (size_t)2 * d * 2, W_up,
                                (size_t)d * 2, (size_t)d * 2, (size_t)dff,
                                cudaMemcpyDeviceToDevice, st));
  }
  DUST_TRY(ensure(ctx, ctx->mlp_dh, (size_t)rows_cap * 2 * d * 2));
  DUST_TRY(ensure(ctx, ctx->part, (size_t)rows_cap * nparts * 4));
  DUST_TRY(ensure(ctx, ctx->dzy, (size_t)rows_cap * 4));
  __nv_bfloat16* da = (__nv_bfloat16*)ctx->mlp_da.p;
  __nv_bfloat16* dh = (__nv_bfloat16*)ctx->mlp_dh.p;
  for (int64_t t0 = 0; t0 < T; t0 += tchunk) {
    const int64_t nt = (t0 + tchunk <= T) ? tchunk : T - t0;
    const int64_t rows = nt * K;
    if (down) {
      DUST_CU(launch_mlp_noise_split(st, p, t0, nt, dh, kTagMlpDown));
      ctx->launches += 1;
    } else if (attn) {
      // sigma eps as planes; du = (sigma eps) W_up^T; da; dh = sigma eps + da W_down^T
      __nv_bfloat16* dn = (__nv_bfloat16*)ctx->mlp_dn.p;
      float* du = (float*)ctx->mlp_du.p;
      DUST_CU(launch_mlp_noise_split(st, p, t0, nt, dn, kTagAttnOut));
      ctx->launches += 1;
      {
        GemmDesc g{};
        g.M = rows; g.N = dff; g.K = 2 * d; g.A = dn; g.lda = 2 * d; g.a_kmajor = true;
        g.B = ctx->wu2.p; g.ldb = 2 * d; g.b_kmajor = true; g.dtype = DUST_BF16;
        EpiDesc e{};
        e.kind = kEpiF32; e.C = du; e.ldc = dff;
        DUST_TRY(run_gemm(ctx, g, e));
      }
      DUST_CU(launch_gelu_delta_rows(st, p, u, du, t0, nt, da));
      ctx->launches += 1;
      GemmDesc g{};
      g.M = rows; g.N = d; g.K = one_plane ? dff : 2 * dff; g.A = da; g.lda = 2 * dff;
      g.a_kmajor = true;
      g.B = one_plane ? W_down : ctx->wd2.p; g.ldb = one_plane ? dff : 2 * dff;
      g.b_kmajor = true; g.dtype = DUST_BF16;
      EpiDesc e{};
      e.kind = kEpiResidSplit; e.Cb = dh; e.ldcb = 2 * d; e.split = d;
      e.resid = dn; e.ldr = 2 * d; e.rsplit = d;
      DUST_TRY(run_gemm(ctx, g, e));
    } else {
      DUST_CU(launch_mlp_delta_a(st, p, u, t0, nt, da, true, nullptr));
      ctx->launches += 1;
      GemmDesc g{};
      g.M = rows; g.N = d; g.K = one_plane ? dff : 2 * dff; g.A = da; g.lda = 2 * dff;
      g.a_kmajor = true;
      g.B = one_plane ? W_down : ctx->wd2.p; g.ldb = one_plane ? dff : 2 * dff;
      g.b_kmajor = true; g.dtype = DUST_BF16;
      EpiDesc e{};
      e.kind = kEpiSplit; e.Cb = dh; e.ldcb = 2 * d; e.split = d;
      DUST_TRY(run_gemm(ctx, g, e));
    }
    // dz = dh_hi W_head^T with the reward epilogue (dz never reaches memory)
    int used_parts = (int)((V + 127) / 128);  // the CUDA-core reward GEMM's 128-column tiles
    {
      GemmDesc g{};
      g.M = rows; g.N = V; g.K = one_plane ? d : 2 * d; g.A = dh; g.lda = 2 * d; g.a_kmajor = true;
      g.B = one_plane ? W_head : ctx->wh2.p; g.ldb = one_plane ? d : 2 * d; g.b_kmajor = true;
      g.dtype = DUST_BF16;
      EpiDesc e{};
      e.kind = kEpiReward; e.P = Z; e.y = targets; e.t0 = t0; e.draws = p.K;
      e.part = (float*)ctx->part.p; e.dzy = (float*)ctx->dzy.p;
      if (ctx->tc_enabled && tc_gemm_supported(g, e)) {
        DUST_TRY(run_gemm(ctx, g, e));
        used_parts = tc_partials_per_row(V);
      } else {
        DUST_CU(launch_reward_gemm_simt(st, g, Z, targets, t0, p.K, (float*)ctx->part.p,
                                        (float*)ctx->dzy.p));
        ctx->launches += 1;
      }
    }
    DUST_CU(launch_reward_combine_rows(st, (float*)ctx->part.p, used_parts, (float*)ctx->dzy.p,
                                       rows, t0 * K, p.K, r));
    ctx->launches += 1;
    if (one_plane) {
      DUST_CU(launch_mlp_reward_corr(st, dh, d, Uw, down ? nullptr : da, dff, Wv, t0, p.K, rows,
                                     r));
      ctx->launches += 1;
    }
  }
  mark(ctx, "perturbed");
  if (attn)
    DUST_CU(launch_noise_g_planes(st, p, r, g_out, (__nv_bfloat16*)ctx->gop.p, kTagAttnOut));
  else
    DUST_CU(launch_mlp_g(st, p, r, g_out, ctx->gop.p, down));
  ctx->launches += 1;
  mark(ctx, "g");
  if (G_out && attn) {
    // G_o = sum_t g_t o_t^T: g as bf16 hi/lo planes against the bf16 O
    DUST_TRY(weight_grad(ctx, p, ctx->gop.p, d, O, d_o, G_out, 0));
    mark(ctx, "gw_gemm");
  } else if (G_out && !down) {
    DUST_TRY(weight_grad(ctx, p, ctx->gop.p, dff, X, d, G_out, 0));
    mark(ctx, "gw_gemm");
  } else if (G_out) {
    // G_down = sum_t g_t a_t^T with a = GELU(u) rounded once to fp32: an fp32
    // contraction over tokens on CUDA cores (2 T d d_ff flops, small next to
    // the perturbed pass)
    DUST_TRY(ensure(ctx, ctx->mlp_a32, (size_t)T * dff * 4));
    DUST_CU(launch_gelu_f32(st, u, T * dff, (float*)ctx->mlp_a32.p, ctx->sm_count));
    ctx->launches += 1;
    dust_params pf = p;
    pf.dtype = DUST_F32;
    DUST_TRY(weight_grad(ctx, pf, ctx->gop.p, d, ctx->mlp_a32.p, dff, G_out, 0));
    mark(ctx, "gw_gemm");
  }
  return finish(ctx, p.flags);
}

dust_status dust_mlp_grad(dust_ctx* ctx, const dust_params* p, const void* X, const void* W_up,
                          const void* W_down, const void* W_head, const int32_t* targets,
                          float* G_up_out, float* loss_out, float* rewards_out, float* g_out) {
  return mlp_impl(ctx, p, kLayerUp, X, nullptr, 0, W_up, W_down, W_head, targets, G_up_out,
                  loss_out, rewards_out, g_out);
}

dust_status dust_mlp_down_grad(dust_ctx* ctx, const dust_params* p, const void* X,
                               const void* W_up, const void* W_down, const void* W_head,
                               const int32_t* targets, float* G_down_out, float* loss_out,
                               float* rewards_out, float* g_out) {
  return mlp_impl(ctx, p, kLayerDown, X, nullptr, 0, W_up, W_down, W_head, targets, G_down_out,
                  loss_out, rewards_out, g_out);
}

dust_status dust_attn_out_grad(dust_ctx* ctx, const dust_params* p, const void* X, const void* O,
                               int64_t d_o, const void* W_up, const void* W_down,
                               const void* W_head, const int32_t* targets, float* G_o_out,
                               float* loss_out, float* rewards_out, float* g_out) {
  return mlp_impl(ctx, p, kLayerAttnOut, X, O, d_o, W_up, W_down, W_head, targets, G_o_out,
                  loss_out, rewards_out, g_out);
}

// Attention internals: noise on the query, key or value projection's output;
// the reward is the first-order loss change -sum_t <o'_t - o_t, e_t> of the
// attention outputs the perturbation moves (k_attn.cu has the closed forms).
dust_status dust_attn_grad(dust_ctx* ctx, const dust_params* pp, const dust_attn_shape* as,
                           const void* X, const float* Q, const float* Kc, const float* Vc,
                           const float* E, float* G_out, float* rewards_out, float* g_out) {
  if (!ctx) return DUST_ERR_ARG;
  char why[256];
  if (check_params(pp, DUST_VARIANT_ATTN, why, sizeof(why)) != DUST_OK)
    return fail(ctx, DUST_ERR_ARG, "%s", why);
  if (!as) return fail(ctx, DUST_ERR_ARG, "shape is NULL");
  const dust_params p = *pp;
  const dust_attn_shape a = *as;
  if (a.which < DUST_ATTN_Q || a.which > DUST_ATTN_V)
    return fail(ctx, DUST_ERR_ARG, "which must be DUST_ATTN_Q, DUST_ATTN_K or DUST_ATTN_V");
  if (a.head_dim != 32 && a.head_dim != 64 && a.head_dim != 128)
    return fail(ctx, DUST_ERR_ARG, "head_dim must be 32, 64 or 128");
  if (a.n_heads < 1 || a.seq_len < 1 || a.seq_len > 4096)
    return fail(ctx, DUST_ERR_ARG, "n_heads must be >= 1 and seq_len in [1, 4096]");
  if (p.T % a.seq_len) return fail(ctx, DUST_ERR_ARG, "T must be a multiple of seq_len");
  if (p.T * a.n_heads >= (1LL << 31)) return fail(ctx, DUST_ERR_ARG, "T * n_heads too large");
  const int64_t T = p.T, H = a.n_heads, Dw = H * (int64_t)a.head_dim, K = p.K;
  if (T > (1LL << 40) / (Dw * K)) return fail(ctx, DUST_ERR_ARG, "T * D * K too large");
  if (!X || !Q || !Kc || !Vc || !E)
    return fail(ctx, DUST_ERR_ARG, "X, Q, K, V and E must be non-NULL");
  if (!aligned(X, 16) || !aligned(Q, 16) || !aligned(Kc, 16) || !aligned(Vc, 16) ||
      !aligned(E, 16) || !aligned(G_out, 4) || !aligned(rewards_out, 4) || !aligned(g_out, 4))
    return fail(ctx, DUST_ERR_ARG, "X, Q, K, V, E must be 16-byte aligned, the outputs 4-byte");
  if ((size_t)ctx->max_smem_optin < attn_fwd_smem(a.seq_len, a.head_dim) ||
      (size_t)ctx->max_smem_optin < attn_draws_smem(a.seq_len, a.head_dim) + 9216 ||
      (size_t)ctx->max_smem_optin < attn_colsum_smem(a.head_dim) ||
      (size_t)ctx->max_smem_optin < (size_t)(Dw + 127) / 128 * 512 + 8192)
    return fail(ctx, DUST_ERR_UNSUPPORTED, "seq_len too long for shared memory");
  DUST_CU(cudaSetDevice(ctx->device));
  const cudaStream_t st = ctx->stream;
  DUST_TRY(ensure(ctx, ctx->attn_o, (size_t)T * Dw * 4));
  DUST_TRY(ensure(ctx, ctx->attn_lse, (size_t)T * H * 4));
  DUST_TRY(ensure(ctx, ctx->attn_gb, (size_t)T * H * 4));
  if (a.which == DUST_ATTN_V)
    DUST_TRY(ensure(ctx, ctx->attn_w, (size_t)T * Dw * 4));
  else
    DUST_TRY(ensure(ctx, ctx->part, (size_t)T * H * K * 4));
  DUST_TRY(ensure(ctx, ctx->gop, gop_bytes(p.dtype, T, Dw)));
  float* r = rewards_out;
  if (!r) {
    DUST_TRY(ensure(ctx, ctx->rew, (size_t)T * K * 4));
    r = (float*)ctx->rew.p;
  }
  DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), st));
  mark(ctx, nullptr);
  float* O = (float*)ctx->attn_o.p;
  float* lse = (float*)ctx->attn_lse.p;
  float* gb = (float*)ctx->attn_gb.p;
  // query and key draws on tensor cores (d_h 64 or 128) unless DUST_ATTN_TC=0
  const char* tc_env = getenv("DUST_ATTN_TC");
  const bool use_tc = a.which != DUST_ATTN_V && a.head_dim >= 64 &&
                      !(tc_env && tc_env[0] == '0') &&
                      (size_t)ctx->max_smem_optin >= attn_tc_smem(a.seq_len, a.head_dim) + 9216;
  if (use_tc) {
    DUST_TRY(ensure(ctx, ctx->attn_tcr, attn_tc_rows_bytes(T, a.seq_len, (int)H, a.head_dim)));
    DUST_TRY(ensure(ctx, ctx->attn_coef, attn_coef_bytes(T, a.seq_len, (int)H)));
  }
  // the clean pass also writes the query-noise coefficient rows, and the
  // key-noise rows when they fit its shared memory (else a pass of their own)
  float2* qcoef = use_tc && a.which == DUST_ATTN_Q ? (float2*)ctx->attn_coef.p : nullptr;
  const bool kfused = use_tc && a.which == DUST_ATTN_K &&
                      (size_t)ctx->max_smem_optin >= attn_fwd_smem(a.seq_len, a.head_dim, true);
  float2* kcoef = kfused ? (float2*)ctx->attn_coef.p : nullptr;
  DUST_CU(launch_attn_fwd(st, T, a.seq_len, (int)H, a.head_dim, Q, Kc, Vc, E, O, lse, gb, qcoef,
                          kcoef));
  ctx->launches += 1;
  mark(ctx, "attn_fwd");
  DUST_CU(launch_attn_draws(st, p, a.which, a.seq_len, (int)H, a.head_dim, Q, Kc, Vc, E, O, lse,
                            gb, (float*)ctx->part.p, (float*)ctx->attn_w.p, r, use_tc,
                            (uint8_t*)ctx->attn_tcr.p, (float2*)ctx->attn_coef.p, kfused,
                            ctx->d_status));
  // value: column sums + draws; tensor cores: (key, unfused) coefficients,
  // row conversion, draws, head sum; CUDA cores: draws, head sum
  ctx->launches += use_tc ? (a.which == DUST_ATTN_K && !kfused ? 4 : 3) : 2;
  mark(ctx, "draws");
  dust_params pg = p;
  pg.d = Dw;  // the noise width
  const int tag = kTagAttnQ + a.which;
  if (p.dtype == DUST_BF16)
    DUST_CU(launch_noise_g_planes(st, pg, r, g_out, (__nv_bfloat16*)ctx->gop.p, tag));
  else
    DUST_CU(launch_noise_g_f32(st, pg, r, g_out, (float*)ctx->gop.p, tag));
  ctx->launches += 1;
  mark(ctx, "g");
  if (G_out) {
    DUST_TRY(weight_grad(ctx, p, ctx->gop.p, Dw, X, p.d, G_out, 0));
    mark(ctx, "gw_gemm");
  }
  return finish(ctx, p.flags);
}

dust_status dust_set_stage_timing(dust_ctx* ctx, int enable) {
  if (!ctx) return DUST_ERR_ARG;
  DUST_CU(cudaSetDevice(ctx->device));
  if (enable && !ctx->ev[0]) {
    for (int i = 0; i < dust_ctx::kMaxMarks; ++i) DUST_CU(cudaEventCreate(&ctx->ev[i]));
  }
  ctx->timing = enable != 0;
  ctx->nmarks = 0;
  return DUST_OK;
}

int dust_stage_times(dust_ctx* ctx, const char** names, float* ms, int cap) {
  if (!ctx || !ctx->timing || ctx->nmarks < 2) return 0;
  cudaSetDevice(ctx->device);
  if (cudaEventSynchronize(ctx->ev[ctx->nmarks - 1]) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const int n = ctx->nmarks - 1;
  for (int i = 0; i < n && i < cap; ++i) {
    float t = 0.0f;
    cudaEventElapsedTime(&t, ctx->ev[i], ctx->ev[i + 1]);
    if (names) names[i] = ctx->mark_name[i + 1];
    if (ms) ms[i] = t;
  }
  return n;
}

int64_t dust_kernel_launches(const dust_ctx* ctx) { return ctx ? ctx->launches : 0; }

dust_status dust_debug_gemm_bf16(dust_ctx* ctx, int64_t M, int64_t N, int64_t K, const void* A,
                                 const void* B, float* C, int path) {
  if (!ctx) return DUST_ERR_ARG;
  if (M < 1 || N < 1 || K < 1 || !A || !B || !C || path < 0 || path > 4)
    return fail(ctx, DUST_ERR_ARG, "bad gemm arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), ctx->stream));
  GemmDesc g{};
  g.M = M; g.N = N; g.K = K; g.A = A; g.lda = K; g.a_kmajor = true;
  g.B = B; g.ldb = K; g.b_kmajor = true; g.dtype = DUST_BF16;
  EpiDesc e{};
  e.kind = kEpiF32; e.C = C; e.ldc = N;
  DUST_TRY(run_gemm(ctx, g, e, path));
  return dust_check(ctx);
}

dust_status dust_debug_gemm_bf16_mn(dust_ctx* ctx, int64_t M, int64_t N, int64_t K, const void* At,
                                    const void* Bt, float* C, int path) {
  if (!ctx) return DUST_ERR_ARG;
  if (M < 1 || N < 1 || K < 1 || !At || !Bt || !C || path < 0 || path > 4)
    return fail(ctx, DUST_ERR_ARG, "bad gemm arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(cudaMemsetAsync(ctx->d_status, 0, sizeof(uint32_t), ctx->stream));
  GemmDesc g{};
  g.M = M; g.N = N; g.K = K; g.A = At; g.lda = M; g.a_kmajor = false;
  g.B = Bt; g.ldb = N; g.b_kmajor = false; g.dtype = DUST_BF16;
  EpiDesc e{};
  e.kind = kEpiF32; e.C = C; e.ldc = N;
  DUST_TRY(run_gemm(ctx, g, e, path));
  return dust_check(ctx);
}

dust_status dust_debug_philox(dust_ctx* ctx, uint64_t seed, const uint32_t* ctr4, int64_t n,
                              uint32_t* out) {
  if (!ctx) return DUST_ERR_ARG;
  if (n < 0 || (n > 0 && (!ctr4 || !out))) return fail(ctx, DUST_ERR_ARG, "bad philox arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(launch_debug_philox(ctx->stream, seed, ctr4, n, out));
  ctx->launches += 1;
  DUST_CU(cudaStreamSynchronize(ctx->stream));
  return DUST_OK;
}

static dust_status debug_gauss_impl(dust_ctx* ctx, const dust_params* p, int32_t tag, int64_t nt,
                                    int64_t ni, int64_t nslots, float* out, int method) {
  if (!ctx) return DUST_ERR_ARG;
  if (!p || nt < 0 || ni < 0 || nslots < 0 || tag < 0 || tag > 255 || !out ||
      p->stream_id >= (1u << 24) || p->token_offset < 0 || p->draw_offset < 0 ||
      p->token_offset + nt > (1LL << 32) || p->draw_offset + ni > (1LL << 32))
    return fail(ctx, DUST_ERR_ARG, "bad gauss arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(launch_debug_gauss(ctx->stream, *p, tag, nt, ni, nslots, out, method));
  ctx->launches += 1;
  DUST_CU(cudaStreamSynchronize(ctx->stream));
  return DUST_OK;
}

dust_status dust_debug_gauss(dust_ctx* ctx, const dust_params* p, int32_t tag, int64_t nt,
                             int64_t ni, int64_t nslots, float* out) {
  return debug_gauss_impl(ctx, p, tag, nt, ni, nslots, out, 0);
}

dust_status dust_debug_gauss_tab(dust_ctx* ctx, const dust_params* p, int32_t tag, int64_t nt,
                                 int64_t ni, int64_t nslots, float* out) {
  return debug_gauss_impl(ctx, p, tag, nt, ni, nslots, out, 1);
}

dust_status dust_debug_gauss_tab_scalar(dust_ctx* ctx, const dust_params* p, int32_t tag,
                                        int64_t nt, int64_t ni, int64_t nslots, float* out) {
  return debug_gauss_impl(ctx, p, tag, nt, ni, nslots, out, 2);
}

dust_status dust_sgd_momentum(dust_ctx* ctx, int64_t n, float lr, float mu, const float* G,
                              float* v, float* W, void* W_bf16) {
  if (!ctx) return DUST_ERR_ARG;
  if (n < 0 || !std::isfinite(lr) || !std::isfinite(mu))
    return fail(ctx, DUST_ERR_ARG, "sgd_momentum: n >= 0 and finite lr, mu are required");
  if (n > 0 && (!G || !v || !W))
    return fail(ctx, DUST_ERR_ARG, "sgd_momentum: G, v and W are required");
  if (!aligned(G, 16) || !aligned(v, 16) || !aligned(W, 16) || !aligned(W_bf16, 8))
    return fail(ctx, DUST_ERR_ARG, "sgd_momentum: G, v, W must be 16-byte and W_bf16 8-byte aligned");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(launch_sgd_momentum(ctx->stream, n, lr, mu, G, v, W, (__nv_bfloat16*)W_bf16,
                              ctx->sm_count));
  ctx->launches += n > 0 ? 1 : 0;
  return DUST_OK;
}

dust_status dust_debug_bm_radius(dust_ctx* ctx, int32_t method, float sigma, float* out) {
  if (!ctx) return DUST_ERR_ARG;
  if (!out || method < 0 || method > 1 || !(sigma >= 0.0f) || !std::isfinite(sigma))
    return fail(ctx, DUST_ERR_ARG, "bad radius arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(launch_debug_bm(ctx->stream, method == 1 ? 3 : 0, sigma, out));
  ctx->launches += 1;
  DUST_CU(cudaStreamSynchronize(ctx->stream));
  return DUST_OK;
}

dust_status dust_debug_bm_angle(dust_ctx* ctx, int32_t method, float* out) {
  if (!ctx) return DUST_ERR_ARG;
  if (!out || method < 0 || method > 1) return fail(ctx, DUST_ERR_ARG, "bad angle arguments");
  DUST_CU(cudaSetDevice(ctx->device));
  DUST_CU(launch_debug_bm(ctx->stream, 1 + method, 0.0f, out));
  ctx->launches += 1;
  DUST_CU(cudaStreamSynchronize(ctx->stream));
  return DUST_OK;
}

}  // extern "C"
