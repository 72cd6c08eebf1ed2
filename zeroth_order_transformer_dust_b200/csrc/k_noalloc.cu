// dust_head_grad_noalloc: the LM-head estimator for callers that cannot call
// cudaMalloc. Such callers include code whose device memory is entirely owned
// by another allocator (a framework's caching allocator or a pre-reserved
// pool, where a fresh cudaMalloc fails or fragments the pool) and
// latency-critical code that cannot afford the device-wide synchronisation
// cudaMalloc and cudaFree can cause. There is no context: every piece of
// scratch (logits, log-sum-exp, partial sums, rewards, the g operand, the
// status word) lives in one file-scope device array of a fixed size that every
// GPU loading this library holds until the process exits. The caller passes
// its inputs and outputs, as with dust_head_grad.
//
// Scope: CUDA-core GEMMs only (the tensor-core path's operand copies would not
// fit a modest array), on the device that is current at the call.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "internal.cuh"

namespace dust {
cudaError_t launch_subset_impl(cudaStream_t st, const dust_params& p, int64_t a, int64_t a_inv,
                               const float* P, const int32_t* y, float* rewards, float* g_out,
                               void* gop, float* gacc, int max_smem_optin);
}  // namespace dust

using namespace dust;

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_base[kMaxDevices] = {};
CUcontext g_ctx[kMaxDevices] = {};

dust_status say(char* msg, int len, dust_status s, const char* fmt, ...) {
  if (msg && len > 0) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, (size_t)len, fmt, ap);
    va_end(ap);
  }
  return s;
}

// The CUDA context current on this thread (NULL if none), through the
// runtime's driver entry-point query, so the library needs no link to the
// driver library itself.
CUcontext current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;  // guarded by g_mu
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuCtxGetCurrent_v4000)ptr;
    else
      cudaGetLastError();
  }
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// Device address of the array on the current device (host code only ever sees
// a host-side stand-in under its name). Looked up once per device and kept
// with the context that was current then; a call under another context (the
// device's primary context destroyed by cudaDeviceReset and created anew)
// looks it up again.
dust_status scratch_base(int dev, void** out, char* msg, int len) {
  if (dev < 0 || dev >= kMaxDevices) return say(msg, len, DUST_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  CUcontext cur = current_context();
  if (!g_base[dev] || !cur || cur != g_ctx[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      cudaGetLastError();
      return say(msg, len, DUST_ERR_CUDA, "cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    }
    cur = current_context();
    g_base[dev] = ptr;
    g_ctx[dev] = cur;
  }
  *out = g_base[dev];
  return DUST_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

struct Carve {
  char* base;
  size_t used = 0;
  void* take(size_t bytes) {
    void* p = base + used;
    used += (bytes + 255) / 256 * 256;
    return p;
  }
};

}  // namespace

extern "C" dust_status dust_head_grad_noalloc(const dust_params* pp, void* cuda_stream,
                                              const void* H, const void* W,
                                              const int32_t* targets, float* G_out,
                                              float* loss_out, float* rewards_out, float* g_out,
                                              char* msg, int msg_len) {
  if (msg && msg_len > 0) msg[0] = 0;
  const dust_status v = dust_validate(pp, DUST_VARIANT_HEAD, msg, msg_len);
  if (v != DUST_OK) return v;
  const dust_params p = *pp;
  if (!H || !W || !targets) return say(msg, msg_len, DUST_ERR_ARG, "H, W and targets must be non-NULL");
  if (!aligned(H, 16) || !aligned(W, 16) || !aligned(targets, 4) || !aligned(G_out, 4) ||
      !aligned(loss_out, 4) || !aligned(rewards_out, 4) || !aligned(g_out, 4))
    return say(msg, msg_len, DUST_ERR_ARG, "H and W must be 16-byte aligned, the other pointers 4-byte");
  const cudaStream_t st = (cudaStream_t)cuda_stream;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return say(msg, msg_len, DUST_ERR_CUDA, "no current CUDA device");
  }
  int max_smem = 0;
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const bool subset = p.S > 0;
  const bool bf16 = p.dtype == DUST_BF16;
  const size_t T = (size_t)p.T, V = (size_t)p.V, K = (size_t)p.K;
  const int nslab = full_vocab_nslab(p.V);

  // scratch plan (each region 256-byte aligned)
  size_t need = 256;                                    // status word
  auto add = [&](size_t b) { need += (b + 255) / 256 * 256; };
  add(T * V * 4);                                       // logits / probabilities
  add(T * 4);                                           // log-sum-exp
  if (!loss_out) add(T * 4);
  if (!subset) {
    if (!rewards_out) add(T * K * 4);
    add(T * (size_t)nslab * K * 4);                      // reward partial sums
    add(full_vocab_xy_bytes(p.T, p.K));                  // noise at the target
  } else {
    add(subset_gacc_bytes(p.T, p.V, max_smem));
  }
  add(bf16 ? 2 * T * V * 2 : T * V * 4);                // g operand
  if (bf16 && G_out) add(2 * T * (size_t)p.d * 2);      // duplicated H
  if (need > kNoAllocScratchBytes)
    return say(msg, msg_len, DUST_ERR_UNSUPPORTED,
               "problem needs %zu bytes of scratch; the static array holds %zu", need,
               kNoAllocScratchBytes);

  void* basev = nullptr;
  const dust_status sb = scratch_base(dev, &basev, msg, msg_len);
  if (sb != DUST_OK) return sb;
  Carve cv{(char*)basev};
  uint32_t* status = (uint32_t*)cv.take(256);
  float* Z = (float*)cv.take(T * V * 4);
  float* lse = (float*)cv.take(T * 4);
  float* loss = loss_out ? loss_out : (float*)cv.take(T * 4);
  float* r = nullptr;
  float* part = nullptr;
  float* xy = nullptr;
  float* gacc = nullptr;
  if (!subset) {
    r = rewards_out ? rewards_out : (float*)cv.take(T * K * 4);
    part = (float*)cv.take(T * (size_t)nslab * K * 4);
    xy = (float*)cv.take(full_vocab_xy_bytes(p.T, p.K));
  } else {
    const size_t gb = subset_gacc_bytes(p.T, p.V, max_smem);
    if (gb) gacc = (float*)cv.take(gb);
  }
  // g operand: bf16 hi/lo planes (2T rows) for bf16 inputs, fp32 otherwise
  const GopFormat gf{bf16 ? kGopBf16Planes : kGopF32, 1.0f};
  void* gop = cv.take(bf16 ? 2 * T * V * 2 : T * V * 4);
  void* xdup = (bf16 && G_out) ? cv.take(2 * T * (size_t)p.d * 2) : nullptr;

  const int64_t a = subset ? subset_stride_of(p) : 0;
  const int64_t a_inv = subset ? modinv(a, p.V) : 0;

  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
  GemmDesc g{};
  g.M = p.T; g.N = p.V; g.K = p.d; g.A = H; g.lda = p.d; g.a_kmajor = true;
  g.B = W; g.ldb = p.d; g.b_kmajor = true; g.b_row_mul = subset ? a : 0; g.dtype = p.dtype;
  EpiDesc ep{};
  ep.kind = kEpiF32; ep.C = Z; ep.ldc = p.V;
  if (e == cudaSuccess) e = launch_gemm_simt(st, g, ep);
  if (e == cudaSuccess)
    e = launch_lse_rows(st, Z, p.T, p.V, targets, subset ? a_inv : 0, lse, loss, subset, status);
  if (!subset) {
    if (e == cudaSuccess) e = launch_full_reward_partial(st, p, Z, lse, targets, part, xy);
    if (e == cudaSuccess) e = launch_full_reward_combine(st, p, part, xy, r);
    if (e == cudaSuccess) e = launch_full_g(st, p, r, g_out, gop, gf);
  } else if (e == cudaSuccess) {
    e = launch_subset_impl(st, p, a, a_inv, Z, targets, rewards_out, g_out, gop, gf, gacc, max_smem);
  }
  if (G_out && e == cudaSuccess) {
    GemmDesc w{};
    EpiDesc we{};
    we.kind = kEpiF32; we.C = G_out; we.ldc = p.d; we.c_row_mul = subset ? a : 0;
    w.M = p.V; w.N = p.d; w.a_kmajor = false; w.b_kmajor = false; w.dtype = p.dtype;
    w.A = gop; w.lda = p.V;
    if (bf16) {
      const size_t hb = T * (size_t)p.d * 2;
      e = cudaMemcpyAsync(xdup, H, hb, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess) e = cudaMemcpyAsync((char*)xdup + hb, H, hb, cudaMemcpyDeviceToDevice, st);
      w.K = 2 * p.T; w.B = xdup; w.ldb = p.d;
    } else {
      w.K = p.T; w.B = H; w.ldb = p.d;
    }
    if (e == cudaSuccess) e = launch_gemm_simt(st, w, we);
  }
  uint32_t hstatus = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&hstatus, status, sizeof(uint32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return say(msg, msg_len, DUST_ERR_CUDA, "CUDA error: %s", cudaGetErrorString(e));
  }
  if (hstatus & kStatusBadTarget) return say(msg, msg_len, DUST_ERR_BOUNDS, "a target lies outside [0, V)");
  return DUST_OK;
}
