// Attention-internals draws ("Dust：无需反向传播的Transformer零阶预训练", §1
// 无需反向传播的信用分配: the attention internals' reward comes from the change
// of the attention output rather than the per-token loss; 减少干扰: only the
// attention output is recomputed per draw, the rest stays cached).
//
// Noise sigma eps on the query, key or value of token s (D = H d_h entries,
// heads side by side) and the reward r = -sum_t <o'_t - o_t, e_t> over the
// tokens whose attention output moves, e the error signal at the attention
// output. Heads do not mix, so r is a sum of per-head rewards r_h, and each
// has a closed form in the clean attention (c = 1/sqrt(d_h), a the clean
// probabilities, gbar_t = <o_t, e_t> per head):
//   query s: row s's scores move by d_tau = c (sigma eps) . k_tau, tau <= s:
//       r_h = -sum_tau a_s,tau expm1(d_tau) (<v_tau, e_s> - gbar_s)
//             / (1 + sum_tau a_s,tau expm1(d_tau));
//   key s:   column s of every row t >= s moves by d_t = c (sigma eps) . q_t;
//       with u_t = a_t,s expm1(d_t) the row's output moves by
//       u_t / (1 + u_t) (v_s - o_t), so
//       r_h = -sum_t u_t / (1 + u_t) (<v_s, e_t> - gbar_t);
//   value s: o_t moves by a_t,s sigma eps, so r_h = -(sigma eps) . w_s with
//       w_s = sum_{t >= s} a_t,s e_t.
// These are exact rewrites of the softmax (nothing is linearised).
//
// B200 mapping: the clean pass is one CTA per (sequence, head, 8 query rows)
// with the rows' keys and values staged through shared memory. The query and
// key draws run one CTA per (token s, head h) and one thread per draw: the
// per-row coefficients (a, <v, e> - gbar) are formed once per CTA, the noise
// of a round of 256 draws once per round, and the keys (query noise) or the
// later queries (key noise) of the sequence stream through 64-row tiles: one
// d_h-long dot product per (draw, row), on tcgen05 in the default form
// (fp16 hi/lo products into TMEM, k_attn_draws_tc) or on the CUDA cores
// (k_attn_draws), then one expm1 and two FMAs on the CUDA cores. Per-head
// rewards go to a (token, head, draw) buffer that a second kernel sums over
// heads in a fixed order. Value noise needs no per-row
// work per draw: w_s = sum_{t >= s} a_t,s e_t comes from one tiled pass (the
// transpose of the clean pass), and each draw is one D-long dot product over
// all heads at once.
#include <cmath>

#include <cuda_fp16.h>

#include "internal.cuh"
#include "noise.cuh"
#include "tc_ptx.cuh"

namespace dust {

size_t attn_fwd_smem(int L, int head_dim, bool kcoef);
size_t attn_colsum_smem(int head_dim);
size_t attn_draws_smem(int L, int head_dim);
size_t attn_tc_smem(int L, int head_dim);
size_t attn_coef_smem(int head_dim);

namespace {

constexpr int kFwdWarps = 8;
constexpr int kDrawThreads = 256;
constexpr int kTile = 64;  // rows per staged tile
constexpr int kTcRows = 64;  // rows per tile of the tensor-core draws: the MMA's N

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// a . b over DH entries (16-byte aligned rows); four partial sums, eight
// float4 pairs in flight at most (the rows come from L2 in the callers).
template <int DH>
__device__ __forceinline__ float dot_row(const float* __restrict__ a, const float* __restrict__ b) {
  float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll 8
  for (int c = 0; c < DH / 4; ++c) {
    const float4 x = reinterpret_cast<const float4*>(a)[c];
    const float4 y = reinterpret_cast<const float4*>(b)[c];
    d0 = fmaf(x.x, y.x, d0);
    d1 = fmaf(x.y, y.y, d1);
    d2 = fmaf(x.z, y.z, d2);
    d3 = fmaf(x.w, y.w, d3);
  }
  return (d0 + d1) + (d2 + d3);
}

// expm1 with full relative accuracy: the Taylor series to x^5 for
// |x| <= 1/16 (truncation below x^5/720 < 2^-29 relative), the library
// function beyond.
__device__ __forceinline__ float expm1_acc(float x) {
  if (fabsf(x) <= 0.0625f) {
    float p = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
    p = fmaf(x, p, 1.0f / 6.0f);
    p = fmaf(x, p, 0.5f);
    p = fmaf(x, p, 1.0f);
    return x * p;
  }
  return expm1f(x);
}

struct FwdArgs {
  const float* Q;
  const float* Kc;
  const float* Vc;
  const float* E;
  float* O;
  float* lse;
  float* gbar;
  int64_t T;
  int32_t L, H;
  float scale;
  float2* qcoef;  // optional: (a_s,tau, a_s,tau <v_tau, e_s>) rows for query noise
  // optional: the key-noise rows, row (s, h) holding at column t of the
  // sequence (a_t,s, <v_s, e_t> - gbar_t) for t >= s (zero for the CTA's rows
  // t < s; entries no CTA writes are cleared by the key draws)
  float2* kcoef = nullptr;
};

// One CTA per (sequence, head, block of kFwdWarps rows), one warp per query
// row t: the causal scores of row t, their log-sum-exp, o_t = sum a v and
// gbar_t = <o_t, e_t>. The CTA's rows share every key and value row, which
// are staged through a shared-memory tile (row stride d_h + 4 floats: the
// lanes' 16-byte reads of different rows fall in distinct banks). Shared
// memory: per warp the row's probabilities (L rounded up to 4) and q_t
// (d_h), and the kTile x (d_h + 4) tile; with key-noise rows also per warp
// <v_s, e_t> for the row's keys (L rounded up to 4) and gbar_t. The key rows
// are written at the end, when gbar_t is known: for each key s of the block
// the CTA's kFwdWarps rows are consecutive columns of row (s, h), 64 bytes.
template <int DH, bool KC>
__device__ __forceinline__ void attn_fwd_body(const FwdArgs& A) {
  extern __shared__ __align__(16) float fsm[];
  constexpr int kStride = DH + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrb = (A.L + kFwdWarps - 1) / kFwdWarps;
  const int rb = blockIdx.x % nrb;
  const int h = (blockIdx.x / nrb) % A.H;
  const int64_t seq = blockIdx.x / ((int64_t)nrb * A.H);
  const int64_t D = (int64_t)A.H * DH;
  const int64_t s0 = seq * A.L;
  const int pos = rb * kFwdWarps + warp;      // this warp's row within the sequence
  const bool row_ok = pos < A.L;
  const int n = row_ok ? pos + 1 : 0;         // keys this row attends to
  const int nmax = min(A.L, (rb + 1) * kFwdWarps);  // keys any row of the CTA needs
  const int Lp = (A.L + 3) & ~3;
  float* pr = fsm + (size_t)warp * (Lp + 2 * DH);
  float* qs = pr + Lp;
  float* es = qs + DH;
  float* tile = fsm + (size_t)kFwdWarps * (Lp + 2 * DH);
  // key rows: <v_s, e_t> per warp (L rounded up to 4), then gbar_t per warp
  float* ev = tile + kTile * kStride + warp * Lp;
  const int64_t t = s0 + pos;
  if (row_ok)
    for (int c = lane; c < DH; c += 32) {
      qs[c] = A.Q[t * D + h * DH + c];
      es[c] = A.E[t * D + h * DH + c];
    }
  // pass 1: scores against staged key tiles
  float m = -INFINITY;
  for (int j0 = 0; j0 < nmax; j0 += kTile) {
    const int rows = min(kTile, nmax - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < rows * (DH / 4); e += kFwdWarps * 32) {
      const int r = e / (DH / 4), c4 = e % (DH / 4);
      *reinterpret_cast<float4*>(tile + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.Kc + (s0 + j0 + r) * D + h * DH)[c4];
    }
    __syncthreads();
    for (int j = lane; j < rows && j0 + j < n; j += 32) {
      const float v = dot_row<DH>(qs, tile + j * kStride) * A.scale;
      pr[j0 + j] = v;
      m = fmaxf(m, v);
    }
  }
  m = warp_max_f(m);
  float l = 0.f;
  for (int j = lane; j < n; j += 32) l += expf(pr[j] - m);
  l = warp_sum_f(l);
  const float lse = m + logf(l);
  for (int j = lane; j < n; j += 32) pr[j] = expf(pr[j] - lse);
  // pass 2: o against staged value tiles
  float o[DH / 32];
#pragma unroll
  for (int u = 0; u < DH / 32; ++u) o[u] = 0.f;
  for (int j0 = 0; j0 < nmax; j0 += kTile) {
    const int rows = min(kTile, nmax - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < rows * (DH / 4); e += kFwdWarps * 32) {
      const int r = e / (DH / 4), c4 = e % (DH / 4);
      *reinterpret_cast<float4*>(tile + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.Vc + (s0 + j0 + r) * D + h * DH)[c4];
    }
    __syncthreads();
    const int lim = min(rows, n - j0);
    for (int j = 0; j < lim; ++j) {
      const float a = pr[j0 + j];
#pragma unroll
      for (int u = 0; u < DH / 32; ++u) o[u] = fmaf(a, tile[j * kStride + lane + 32 * u], o[u]);
    }
    if (KC)
      for (int j = lane; j < lim; j += 32) ev[j0 + j] = dot_row<DH>(es, tile + j * kStride);
    if (A.qcoef && row_ok) {
      // the query-noise coefficient row: (a, a <v, e_s>) up to the tile
      // boundary, zero past the causal limit (<o_s, e_s> is taken off later)
      const int Lt = (A.L + kTcRows - 1) / kTcRows * kTcRows;
      float2* crow = A.qcoef + (t * A.H + h) * (int64_t)Lt + j0;
      for (int j = lane; j < kTile; j += 32) {
        float2 v = make_float2(0.f, 0.f);
        if (j < lim) {
          const float a = pr[j0 + j];
          v = make_float2(a, a * dot_row<DH>(es, tile + j * kStride));
        }
        crow[j] = v;
      }
    }
  }
  float gb = 0.f;
  if (row_ok) {
#pragma unroll
    for (int u = 0; u < DH / 32; ++u) {
      const int64_t c = t * D + h * DH + lane + 32 * u;
      A.O[c] = o[u];
      gb = fmaf(o[u], A.E[c], gb);
    }
    gb = warp_sum_f(gb);
    if (lane == 0) {
      A.lse[t * A.H + h] = lse;
      A.gbar[t * A.H + h] = gb;
    }
  }
  if (!KC) return;
  const float* evs = tile + kTile * kStride;
  float* gbs = const_cast<float*>(evs) + kFwdWarps * Lp;
  if (lane == 0) gbs[warp] = gb;
  __syncthreads();
  // key rows: entry e = (key s, warp w), w fastest, so every 8 threads write
  // columns rb kFwdWarps .. + 7 of row (s, h)
  const int Lt = (A.L + kTcRows - 1) / kTcRows * kTcRows;
  float2* kbase = A.kcoef + (s0 * A.H + h) * (int64_t)Lt + rb * kFwdWarps;
  for (int e = threadIdx.x; e < nmax * kFwdWarps; e += kFwdWarps * 32) {
    const int w = e % kFwdWarps, sk = e / kFwdWarps;
    const int c = rb * kFwdWarps + w;  // the row (query position) of warp w
    float2 v = make_float2(0.f, 0.f);
    if (c < A.L && sk <= c)
      v = make_float2(fsm[w * (Lp + 2 * DH) + sk], evs[w * Lp + sk] - gbs[w]);
    if (c < Lt) kbase[(int64_t)sk * A.H * Lt + w] = v;
  }
}

template <int DH>
__global__ __launch_bounds__(kFwdWarps * 32) void k_attn_fwd(const __grid_constant__ FwdArgs A) {
  attn_fwd_body<DH, false>(A);
}

// The clean pass that also writes the key-noise rows. Its shared memory
// (the extra <v_s, e_t> rows) allows two CTAs per SM, and so do its
// registers: with that bound ptxas keeps every value in registers.
template <int DH>
__global__ __launch_bounds__(kFwdWarps * 32, 2) void k_attn_fwd_kc(const __grid_constant__ FwdArgs A) {
  attn_fwd_body<DH, true>(A);
}

struct DrawArgs {
  const float* Q;
  const float* Kc;
  const float* Vc;
  const float* E;
  const float* O;
  const float* lse;
  const float* gbar;
  float* part;  // (T H) x K: r_h of (token, head) for every draw
  RoundKeys keys;
  uint32_t t_off, i_off, ctr3;
  float xscale;  // sigma c (query, key) or sigma (value): the noise's factor
  int64_t T;
  int32_t L, H, K;
  float scale;
};

// Noise of head h for kDrawThreads draws of token s, times the table's
// factor, into xs[draw * (d_h + 1) + j] (the odd row stride keeps the
// per-thread row reads free of bank conflicts). Slot h d_h + j of the layer's
// D slots uses counter (slot_ctr0(slot >> 7, slot & 31), t, i, ctr3), word
// (slot >> 5) & 3; words (0, 1) and (2, 3) are the two Box-Muller pairs of a
// counter. For d_h >= 64 the head's 32-slot groups pair up within one counter
// (one transform gives both); a 32-wide head uses one word of a pair. Work
// item (draw, lane, group pair) per thread, so no thread holds a row.
template <int DH>
__device__ __forceinline__ void head_noise_smem(float* xs, const RoundKeys& keys, uint32_t t_abs,
                                                uint32_t i_off, int i0, int K, uint32_t ctr3,
                                                int h, const float2* tab) {
  constexpr int kPairs = DH >= 64 ? DH / 64 : 1;
  const int items = kDrawThreads * 32 * kPairs;
  for (int it = threadIdx.x; it < items; it += kDrawThreads) {
    const int l = it & 31;
    const int rest = it >> 5;
    const int pr = rest % kPairs;
    const int d = rest / kPairs;  // draw within the round
    const int i = i0 + d;
    if (i >= K) {  // no draw: zero noise, so the pair's shuffles see finite values
      for (int q = 0; q < (DH >= 64 ? 2 : 1); ++q)
        xs[d * (DH + 1) + (DH >= 64 ? 64 * pr + 32 * q : 0) + l] = 0.0f;
      continue;
    }
    const DrawConst dc = draw_const(keys, t_abs, i_off + (uint32_t)i);
    const uint32_t sb = (uint32_t)h * DH + 64u * pr;
    const uint32_t blk = sb >> 7, word = (sb >> 5) & 3u;
    const U4 w = philox_from2(block_const(keys, slot_ctr0(blk, (uint32_t)l), ctr3), dc, keys);
    const float2 nn = box_muller_tab(word >= 2 ? w.z : w.x, word >= 2 ? w.w : w.y, tab);
    float* row = xs + d * (DH + 1);
    if (DH >= 64) {
      row[64 * pr + l] = nn.x;
      row[64 * pr + 32 + l] = nn.y;
    } else {
      row[l] = (word & 1u) ? nn.y : nn.x;
    }
  }
}

// One CTA per (token s, head h): blockIdx.x = s H + h. WHICH: 0 query,
// 1 key. Dynamic shared memory: the per-row coefficient pairs (L
// float2, L rounded up to 4), a kTile x (d_h + 8) tile and the noise rows of
// one round of kDrawThreads draws.
template <int WHICH, int DH>
__global__ __launch_bounds__(kDrawThreads, DH <= 64 ? 2 : 1) void k_attn_draws(const __grid_constant__ DrawArgs A) {
  extern __shared__ __align__(16) float dsm[];
  __shared__ float2 tab[kSinCosTable];
  __shared__ __align__(16) float own[2][DH];
  const int tid = threadIdx.x;
  const int64_t s = blockIdx.x / A.H;
  const int h = (int)(blockIdx.x % A.H);
  const int64_t D = (int64_t)A.H * DH;
  const int64_t s0 = s - s % A.L;
  // the other index runs over tau in [s0, s] (query) or t in [s, s0 + L) (key)
  const int64_t r0 = WHICH == 0 ? s0 : s;
  const int n = WHICH == 0 ? (int)(s - s0) + 1 : (int)(s0 + A.L - s);
  const int Lp = (A.L + 3) & ~3;
  // a tile row holds the two halves of d_h with 4 floats between them, so the
  // pair's two 16-byte reads fall in different banks
  constexpr int kTileStride = DH + 8;
  float2* cab = reinterpret_cast<float2*>(dsm);  // per row: (a, b) or (a, beta)
  float* tile = dsm + 2 * Lp;
  float* xs = tile + kTile * kTileStride;
  fill_sincos_table(tab, A.xscale);
  for (int c = tid; c < DH; c += kDrawThreads) {
    const int64_t o = s * D + h * DH + c;
    own[0][c] = WHICH == 0 ? A.Q[o] : A.Kc[o];
    own[1][c] = WHICH == 0 ? A.E[o] : A.Vc[o];
  }
  __syncthreads();
  // per-row coefficients, once per CTA
  const float lse_s = A.lse[s * A.H + h];
  const float gb_s = A.gbar[s * A.H + h];
  for (int j = tid; j < n; j += kDrawThreads) {
    const int64_t row = (r0 + j) * D + h * DH;
    if (WHICH == 0) {
      const float a = expf(dot_row<DH>(own[0], A.Kc + row) * A.scale - lse_s);
      cab[j] = make_float2(a, a * (dot_row<DH>(own[1], A.Vc + row) - gb_s));
    } else {
      const int64_t t = r0 + j;
      const float a = expf(dot_row<DH>(own[0], A.Q + row) * A.scale - A.lse[t * A.H + h]);
      cab[j] = make_float2(a, dot_row<DH>(own[1], A.E + row) - A.gbar[t * A.H + h]);
    }
  }
  __syncthreads();
  const uint32_t t_abs = A.t_off + (uint32_t)s;
  const float* src = WHICH == 0 ? A.Kc : A.Q;  // rows streamed through the tile
  for (int i0 = 0; i0 < A.K; i0 += kDrawThreads) {
    const int i = i0 + tid;
    const bool live = i < A.K;
    __syncthreads();  // the previous round's rows are consumed
    head_noise_smem<DH>(xs, A.keys, t_abs, A.i_off, i0, A.K, A.ctr3, h, tab);
    __syncthreads();
    float r;
    {
      // Thread pairs: both threads of a pair hold the noise of the pair's two
      // draws, each for one half of the head's dims, so every 16-byte tile
      // read feeds eight multiply-adds; one shuffle completes the dot product
      // of the thread's own draw (tid) from the two halves.
      constexpr int HD = DH / 2;
      const int half = tid & 1;
      const float* xa_row = xs + (tid & ~1) * (DH + 1) + half * HD;
      float xa[HD], xb[HD];
#pragma unroll
      for (int c = 0; c < HD; ++c) {
        xa[c] = xa_row[c];
        xb[c] = xa_row[DH + 1 + c];
      }
      float acc0 = 0.f, acc1 = 0.f;
      for (int j0 = 0; j0 < n; j0 += kTile) {
        const int m = min(kTile, n - j0);
        __syncthreads();
        for (int e = tid; e < m * (DH / 4); e += kDrawThreads) {
          const int row = e / (DH / 4), c4 = e % (DH / 4);
          const int dst = row * kTileStride + 4 * c4 + (4 * c4 >= HD ? 4 : 0);
          *reinterpret_cast<float4*>(tile + dst) =
              reinterpret_cast<const float4*>(src + (r0 + j0 + row) * D + h * DH)[c4];
        }
        __syncthreads();
#pragma unroll 2
        for (int jj = 0; jj < m; ++jj) {
          const float* tr = tile + jj * kTileStride + half * (HD + 4);
          float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
          for (int c = 0; c < HD; c += 4) {
            const float4 v = *reinterpret_cast<const float4*>(tr + c);
            a0 = fmaf(xa[c], v.x, a0);
            b0 = fmaf(xb[c], v.x, b0);
            a1 = fmaf(xa[c + 1], v.y, a1);
            b1 = fmaf(xb[c + 1], v.y, b1);
            a0 = fmaf(xa[c + 2], v.z, a0);
            b0 = fmaf(xb[c + 2], v.z, b0);
            a1 = fmaf(xa[c + 3], v.w, a1);
            b1 = fmaf(xb[c + 3], v.w, b1);
          }
          const float pa = a0 + a1, pb = b0 + b1;
          const float dot = (half ? pb : pa) + __shfl_xor_sync(0xffffffffu, half ? pa : pb, 1);
          const float em = expm1_acc(dot);
          const float2 cf = cab[j0 + jj];
          if (WHICH == 0) {
            acc0 = fmaf(cf.x, em, acc0);
            acc1 = fmaf(cf.y, em, acc1);
          } else {
            const float u = cf.x * em;
            acc1 = fmaf(__fdividef(u, 1.0f + u), cf.y, acc1);
          }
        }
      }
      r = WHICH == 0 ? -acc1 / (1.0f + acc0) : -acc1;
    }
    if (live) A.part[(int64_t)blockIdx.x * A.K + i] = r;
  }
}

// Per-row coefficients of the key draws, for every (token s, head h) at
// once: row (s, h) of C holds, at column c of s's sequence (c < the sequence
// length rounded up to 64), (a_c,s, <v_s, e_c> - gbar_c) for c >= pos(s) and
// zero before (the query draws' rows come from the clean pass). One CTA per
// (sequence, head, block of kFwdWarps key positions s), one warp per s; the
// later queries and their error rows are staged in shared-memory tiles (row
// stride d_h + 4) shared by the CTA's warps, each lane takes tile rows lane
// and lane + 32, and the row's writes are coalesced float2 stores.
template <int DH>
__global__ __launch_bounds__(kFwdWarps * 32) void k_attn_kcoef(const __grid_constant__ FwdArgs A,
                                                              float2* __restrict__ C) {
  extern __shared__ __align__(16) float qsm[];
  constexpr int kStride = DH + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrb = (A.L + kFwdWarps - 1) / kFwdWarps;
  const int rb = blockIdx.x % nrb;
  const int h = (blockIdx.x / nrb) % A.H;
  const int64_t seq = blockIdx.x / ((int64_t)nrb * A.H);
  const int64_t D = (int64_t)A.H * DH;
  const int64_t s0 = seq * A.L;
  const int Lt = (A.L + kTcRows - 1) / kTcRows * kTcRows;
  const int pos = rb * kFwdWarps + warp;
  const bool ok = pos < A.L;
  float* tq = qsm;                          // queries of the tile rows
  float* te = tq + kTile * kStride;         // their error signals
  float* lt = te + kTile * kStride;         // their LSE
  float* gt = lt + kTile;                   // and <o, e>
  float* own = gt + kTile + (size_t)warp * 2 * DH;  // k_s, v_s
  const int64_t so = (s0 + pos) * D + h * DH;
  if (ok)
    for (int c = lane; c < DH; c += 32) {
      own[c] = A.Kc[so + c];
      own[DH + c] = A.Vc[so + c];
    }
  // columns [pos, L) of each row, from the block's first whole tile
  const int c_lo = rb * kFwdWarps / kTcRows * kTcRows;
  float2* crow = C + ((s0 + pos) * A.H + h) * (int64_t)Lt;
  for (int j0 = c_lo; j0 < Lt; j0 += kTile) {
    const int rows = min(kTile, A.L - j0);  // rows past the sequence end stay unread
    __syncthreads();
    for (int e = threadIdx.x; e < rows * (DH / 4); e += kFwdWarps * 32) {
      const int r = e / (DH / 4), c4 = e % (DH / 4);
      const int64_t src = (s0 + j0 + r) * D + h * DH;
      *reinterpret_cast<float4*>(tq + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.Q + src)[c4];
      *reinterpret_cast<float4*>(te + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.E + src)[c4];
    }
    for (int r = threadIdx.x; r < rows; r += kFwdWarps * 32) {
      lt[r] = A.lse[(s0 + j0 + r) * A.H + h];
      gt[r] = A.gbar[(s0 + j0 + r) * A.H + h];
    }
    __syncthreads();
    if (ok) {
      for (int j = lane; j < kTile; j += 32) {
        const int c = j0 + j;
        float2 v = make_float2(0.f, 0.f);
        if (c < A.L && c >= pos) {
          const float a = expf(dot_row<DH>(own, tq + j * kStride) * A.scale - lt[j]);
          v = make_float2(a, dot_row<DH>(own + DH, te + j * kStride) - gt[j]);
        }
        crow[c] = v;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Tensor-core form of the query/key draws (d_h = 64 or 128). Per (token s,
// head h) and round of 256 draws, the (draw x row) dot products are the
// product X R^T of the draws' noise X (256 x d_h) and the streamed rows R
// (64 x d_h per tile). Both are split into fp16 hi + lo parts and the product
// is taken as X_hi R_hi + X_hi R_lo + X_lo R_hi, with fp32 accumulation in
// TMEM: the dropped X_lo R_lo term is 2^-22 of |x| |r|. The noise carries a
// power-of-two factor S (in the Box-Muller table) that keeps its lo parts
// normal in fp16; the epilogue divides it out. One thread issues the MMAs
// (M = 128 per half of the draws, N = 64, K = 16 per instruction, operands
// K-major in 128-byte-swizzled shared memory tiles written by the threads);
// every thread then reads its own draw's 64 dot products from TMEM and runs
// the expm1 epilogue of the CUDA-core kernel. TMEM and the row tiles are
// double buffered and handed over through mbarriers, without block barriers
// inside a round: thread 0 bulk-copies row tile j + 2 while the epilogue of
// tile j runs, and issues the MMAs of tile j + 1 once its rows have landed
// (full) and the epilogue of tile j - 1 has read its TMEM buffer (empty, one
// arrival per warp); the epilogue waits for its tile's MMAs (done).
constexpr int kTcTmemCols = 256;    // 2 buffers x 2 halves of the draws x 64 columns
constexpr uint64_t kTcWaitNs = 2000000000ull;

struct TcDrawArgs {
  const float* gbar;    // <o, e> per (token, head)
  float* part;
  const uint8_t* rows;  // the streamed rows, converted (k_attn_tc_rows)
  const float2* coef;   // the per-row coefficients, rows of Lt
  RoundKeys keys;
  uint32_t t_off, i_off, ctr3;
  float xscale;  // sigma c S: the noise's factor
  float inv_s;   // 1 / S
  int64_t T;
  int32_t L, H, K;
  uint32_t* status;
};

// Byte offset of fp16 element (row, col) of a K-major tile of 64 columns with
// 128-byte swizzling: 16-byte chunk c of row r sits at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128_off(int row, int col) {
  return (uint32_t)row * 128u + ((((uint32_t)col >> 3) ^ ((uint32_t)row & 7u)) << 4) +
         ((uint32_t)col & 7u) * 2u;
}

template <int DH>
struct TcLayout {
  static constexpr int KB = DH / 64;                      // 64-column K blocks
  static constexpr uint32_t A_TILE = 128 * 128;           // 128 rows x 64 fp16
  static constexpr uint32_t B_TILE = kTcRows * 128;       // 64 rows x 64 fp16
  static constexpr uint32_t A_BYTES = 2 * 2 * KB * A_TILE;  // [half][hi, lo][kb]
  static constexpr uint32_t B_BYTES = 2 * 2 * KB * B_TILE;  // [buffer][hi, lo][kb]
  __host__ __device__ static constexpr uint32_t a_off(int mh, int part, int kb) {
    return ((uint32_t)(mh * 2 + part) * KB + kb) * A_TILE;
  }
  __host__ __device__ static constexpr uint32_t b_off(int buf, int part, int kb) {
    return A_BYTES + ((uint32_t)(buf * 2 + part) * KB + kb) * B_TILE;
  }
};

// Bounded mbarrier wait: gives up after kTcWaitNs, or at once when another
// thread of the CTA has given up (abort), setting the abort flag and the
// timeout bit of the status word.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                        uint32_t* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (ptx::globaltimer_ns() - t0 > kTcWaitNs) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// The round's noise (draws i0 .. i0 + 255, head h), times S, as fp16 hi and
// lo parts in the A tiles. Work item (draw, lane, 64-slot group): one counter
// and one Box-Muller pair give channels 64 g + lane and 64 g + 32 + lane.
template <int DH>
__device__ __forceinline__ void tc_noise(uint8_t* sm, const TcDrawArgs& A, uint32_t t_abs, int i0,
                                         int h) {
  using Ly = TcLayout<DH>;
  for (int it = threadIdx.x; it < kDrawThreads * 32 * Ly::KB; it += kDrawThreads) {
    const int l = it & 31;
    const int rest = it >> 5;
    const int g = rest % Ly::KB;
    const int d = rest / Ly::KB;
    float v0 = 0.f, v1 = 0.f;
    if (i0 + d < A.K) {
      const DrawConst dc = draw_const(A.keys, t_abs, A.i_off + (uint32_t)(i0 + d));
      const uint32_t sb = (uint32_t)h * DH + 64u * g;
      const bool hi_pair = ((sb >> 5) & 3u) != 0u;
      const U4 w = philox_from2(block_const(A.keys, slot_ctr0(sb >> 7, (uint32_t)l), A.ctr3), dc,
                                A.keys);
      const float2 nn = box_muller(hi_pair ? w.z : w.x, hi_pair ? w.w : w.y, A.xscale);
      v0 = nn.x;
      v1 = nn.y;
    }
    const int r = d & 127, mh = d >> 7;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float v = q ? v1 : v0;
      const __half hi = __float2half_rn(v);
      const __half lo = __float2half_rn(v - __half2float(hi));
      const uint32_t o = sw128_off(r, 32 * q + l);
      *reinterpret_cast<__half*>(sm + Ly::a_off(mh, 0, g) + o) = hi;
      *reinterpret_cast<__half*>(sm + Ly::a_off(mh, 1, g) + o) = lo;
    }
  }
}

// The streamed rows (keys for query noise, queries for key noise) as fp16
// hi and lo parts, converted once per call into the B-tile layout: for each
// (sequence, head, 64-row tile of the sequence) the tiles [hi | lo] x K
// blocks, 16 KB per 64 head dims, rows past the sequence end zero. Values
// beyond +-32768 set kStatusRange. One CTA per tile.
template <int DH>
__global__ __launch_bounds__(kDrawThreads) void k_attn_tc_rows(const float* __restrict__ src,
                                                               int64_t T, int32_t L, int32_t H,
                                                               uint8_t* __restrict__ out,
                                                               uint32_t* status) {
  using Ly = TcLayout<DH>;
  const int ntile = (L + kTcRows - 1) / kTcRows;
  const int64_t unit = blockIdx.x;  // ((seq H) + h) ntile + k
  const int k = (int)(unit % ntile);
  const int h = (int)((unit / ntile) % H);
  const int64_t seq = unit / ((int64_t)ntile * H);
  const int64_t D = (int64_t)H * DH;
  uint8_t* dst = out + (size_t)unit * 2 * Ly::KB * Ly::B_TILE;
  bool bad = false;
  for (int e = threadIdx.x; e < kTcRows * (DH / 4); e += kDrawThreads) {
    const int r = e / (DH / 4), c = 4 * (e % (DH / 4));
    const int pos = k * kTcRows + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (pos < L) v = *reinterpret_cast<const float4*>(src + (seq * L + pos) * D + h * DH + c);
    const float f[4] = {v.x, v.y, v.z, v.w};
    __half hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      bad |= !(fabsf(f[q]) < 32768.0f);
      hi[q] = __float2half_rn(f[q]);
      lo[q] = __float2half_rn(f[q] - __half2float(hi[q]));
    }
    const int kb = c >> 6, col = c & 63;
    const uint32_t o = sw128_off(r, col);
    *reinterpret_cast<uint2*>(dst + (size_t)kb * Ly::B_TILE + o) =
        make_uint2(((uint32_t)__half_as_ushort(hi[1]) << 16) | __half_as_ushort(hi[0]),
                   ((uint32_t)__half_as_ushort(hi[3]) << 16) | __half_as_ushort(hi[2]));
    *reinterpret_cast<uint2*>(dst + (size_t)(Ly::KB + kb) * Ly::B_TILE + o) =
        make_uint2(((uint32_t)__half_as_ushort(lo[1]) << 16) | __half_as_ushort(lo[0]),
                   ((uint32_t)__half_as_ushort(lo[3]) << 16) | __half_as_ushort(lo[2]));
  }
  if (bad) atomicOr(status, kStatusRange);
}

// The MMAs of one tile into TMEM buffer `buf`: for each half of the draws,
// X_hi R_hi + X_hi R_lo + X_lo R_hi over the K blocks, 16 columns per MMA.
template <int DH>
__device__ __forceinline__ void tc_issue(uint32_t base, uint32_t tmem, int buf, uint32_t bar) {
  using Ly = TcLayout<DH>;
  constexpr uint32_t idesc = ptx::idesc_f16_f32(128, kTcRows);
#pragma unroll
  for (int mh = 0; mh < 2; ++mh) {
    const uint32_t d = tmem + (uint32_t)(buf * 128 + mh * 64);
    uint32_t accum = 0;
#pragma unroll
    for (int kb = 0; kb < Ly::KB; ++kb)
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        const uint32_t a = base + Ly::a_off(mh, term == 2 ? 1 : 0, kb);
        const uint32_t b = base + Ly::b_off(buf, term == 1 ? 1 : 0, kb);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ptx::mma_f16(d, ptx::sdesc_kmajor_sw128(a + 32u * k), ptx::sdesc_kmajor_sw128(b + 32u * k),
                       idesc, accum);
          accum = 1;
        }
      }
  }
  ptx::mma_commit(bar);
}

// The epilogue of 32 columns with the exact expm1 (a product beyond
// |x| = 1/16 among them): reads the columns from TMEM again, out of line so
// that the common path keeps its registers. Called by whole warps.
template <int WHICH>
__device__ __noinline__ float2 tc_exact_chunk(uint32_t taddr, const float2* cf, float inv_s) {
  float v[32];
  ptx::tmem_ld32(taddr, v);
  float c0 = 0.f, c1 = 0.f;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float em = expm1_acc(v[q] * inv_s);
    const float2 c = cf[q];
    if (WHICH == 0) {
      c0 = fmaf(c.x, em, c0);
      c1 = fmaf(c.y, em, c1);
    } else {
      const float u = c.x * em;
      c1 = fmaf(__fdividef(u, 1.0f + u), c.y, c1);
    }
  }
  return make_float2(c0, c1);
}

// One CTA per (token s, head h), as k_attn_draws; thread tid is draw i0 + tid
// of each round, and TMEM lane (tid & 127) of the draws' half tid >> 7.
template <int WHICH, int DH>
__global__ __launch_bounds__(kDrawThreads, DH == 64 ? 2 : 1) void k_attn_draws_tc(const __grid_constant__ TcDrawArgs A) {
  using Ly = TcLayout<DH>;
  extern __shared__ uint8_t tsm_raw[];
  __shared__ __align__(8) uint64_t full[2], done[2], empty[2], cfull;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t raw = ptx::smem_u32(tsm_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = tsm_raw + (base - raw);
  float2* cab = reinterpret_cast<float2*>(sm + Ly::A_BYTES + Ly::B_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t s = blockIdx.x / A.H;
  const int h = (int)(blockIdx.x % A.H);
  const int64_t s0 = s - s % A.L;
  // rows streamed: tau in [s0, s] (query noise) or t in [s, s0 + L) (key
  // noise), in the converted 64-row tiles of the sequence: from tile k0 on,
  // with zero coefficients for the rows of tile k0 before s (key noise)
  const int k0 = WHICH == 0 ? 0 : (int)((s - s0) / kTcRows);
  const int64_t r0 = s0 + (int64_t)k0 * kTcRows;
  const int n = WHICH == 0 ? (int)(s - s0) + 1 : (int)(s0 + A.L - r0);
  const int ntile_seq = (A.L + kTcRows - 1) / kTcRows;
  const uint8_t* tiles = A.rows + ((size_t)(s / A.L) * A.H + h) * ntile_seq * (2 * Ly::KB * Ly::B_TILE) +
                         (size_t)k0 * (2 * Ly::KB * Ly::B_TILE);
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&full[b]), 1);
      ptx::mbar_init(ptx::smem_u32(&done[b]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[b]), kDrawThreads / 32);
    }
    ptx::mbar_init(ptx::smem_u32(&cfull), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(&tmem_slot), kTcTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  // the coefficient row of (s, h) from column r0 - s0 on, whole tiles, by
  // bulk copy: it lands while the round's noise is drawn
  if (tid == 0) {
    const int Lt = (A.L + kTcRows - 1) / kTcRows * kTcRows;
    const float2* crow = A.coef + (s * A.H + h) * (int64_t)Lt + (r0 - s0);
    const uint32_t bytes = (uint32_t)((n + kTcRows - 1) / kTcRows * kTcRows) * 8u;
    const uint32_t cb = ptx::smem_u32(&cfull);
    ptx::mbar_expect_tx(cb, bytes);
    ptx::bulk_load(ptx::smem_u32(cab), crow, bytes, cb);
  }
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int ntiles = (n + kTcRows - 1) / kTcRows;
  constexpr uint32_t kTileBytes = 2 * Ly::KB * Ly::B_TILE;
  const int mh = warp >> 2, quad = warp & 3;
  const uint32_t tlane = (uint32_t)(quad * 32) << 16;
  const uint32_t t_abs = A.t_off + (uint32_t)s;
  const float gb_s = WHICH == 0 ? A.gbar[s * A.H + h] : 0.f;  // <o_s, e_s>
  volatile int* abort = &abort_flag;
  // parities of the next completion of full/done/empty[b] (bit b); uses of
  // each TMEM buffer so far (its first use needs no empty wait)
  uint32_t pf = 0, pd = 0, pe = 0, used = 0;
  auto copy_tile = [&](int j) {  // thread 0: row tile j into B buffer j & 1
    const uint32_t fb = ptx::smem_u32(&full[j & 1]);
    ptx::mbar_expect_tx(fb, kTileBytes);
    ptx::bulk_load(base + Ly::b_off(j & 1, 0, 0), tiles + (size_t)j * kTileBytes, kTileBytes, fb);
  };
  auto issue = [&](int j) -> bool {  // thread 0: the MMAs of tile j
    const int b = j & 1;
    if (!tc_wait(ptx::smem_u32(&full[b]), (pf >> b) & 1u, abort, A.status)) return false;
    pf ^= 1u << b;
    if (used & (1u << b)) {
      if (!tc_wait(ptx::smem_u32(&empty[b]), (pe >> b) & 1u, abort, A.status)) return false;
      pe ^= 1u << b;
    }
    used |= 1u << b;
    ptx::tc_fence_after();
    tc_issue<DH>(base, tmem, b, ptx::smem_u32(&done[b]));
    return true;
  };
  for (int i0 = 0; i0 < A.K && !*abort; i0 += kDrawThreads) {
    if (tid == 0) {
      copy_tile(0);
      if (ntiles > 1) copy_tile(1);
    }
    tc_noise<DH>(sm, A, t_abs, i0, h);
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();  // the round's noise is in place; the last round's epilogues are done
    ptx::tc_fence_after();
    // a failed wait sets the abort flag; every thread still reaches the next
    // done-wait, and the warps leave the tile loop warp-uniformly
    if (tid == 0) issue(0);
    // the coefficient row (phase 0 of cfull: at once in later rounds); a
    // failure sets the abort flag, which ends the tile loop below
    (void)__all_sync(0xffffffffu, tc_wait(ptx::smem_u32(&cfull), 0u, abort, A.status));
    if (WHICH == 1 && i0 == 0) {
      // key rows: the entries of tile k0 before s and those past the
      // sequence end carry no coefficient (the clean pass that writes the
      // rows leaves some of them unwritten); clear them once
      const int before = (int)(s - r0);
      for (int q = tid; q < ntiles * kTcRows; q += kDrawThreads)
        if (q < before || q >= n) cab[q] = make_float2(0.f, 0.f);
      __syncthreads();
    }
    float acc0 = 0.f, acc1 = 0.f;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      if (tid == 0 && j + 1 < ntiles) issue(j + 1);
      const bool got = tc_wait(ptx::smem_u32(&done[b]), (pd >> b) & 1u, abort, A.status);
      if (!__all_sync(0xffffffffu, got)) break;  // the warp converges here (tcgen05.ld is .aligned)
      pd ^= 1u << b;
      ptx::tc_fence_after();
      // rows beyond n of a partial tile are zero rows of B with zero
      // coefficients (cab is zero-filled up to the tile boundary), so every
      // tile runs all 64 columns, 32 at a time
      const uint32_t ta = tmem + tlane + (uint32_t)(b * 128 + mh * 64);
#pragma unroll 1
      for (int hc = 0; hc < 2; ++hc) {
        float v[32];
        ptx::tmem_ld32(ta + 32u * hc, v);
        const float2* cf = cab + j * kTcRows + 32 * hc;
        // the degree-5 series of expm1 without a branch per element; a
        // product beyond |x| = 1/16 (rare at the usual sigma) sends the
        // warp's 32 columns through the exact form instead
        float c0 = 0.f, c1 = 0.f;
        bool wide = false;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float x = v[q] * A.inv_s;
          wide |= fabsf(x) > 0.0625f;
          float pp = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
          pp = fmaf(x, pp, 1.0f / 6.0f);
          pp = fmaf(x, pp, 0.5f);
          pp = fmaf(x, pp, 1.0f);
          const float em = x * pp;
          const float2 c = cf[q];
          if (WHICH == 0) {
            c0 = fmaf(c.x, em, c0);
            c1 = fmaf(c.y, em, c1);
          } else {
            const float u = c.x * em;
            c1 = fmaf(__fdividef(u, 1.0f + u), c.y, c1);
          }
        }
        if (__any_sync(0xffffffffu, wide)) {  // warp-uniform
          const float2 cc = tc_exact_chunk<WHICH>(ta + 32u * hc, cf, A.inv_s);
          c0 = cc.x;
          c1 = cc.y;
        }
        acc0 += c0;
        acc1 += c1;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) ptx::mbar_arrive(ptx::smem_u32(&empty[b]));
      // B buffer b is free again (the MMAs of tile j are done): tile j + 2
      if (tid == 0 && j + 2 < ntiles) copy_tile(j + 2);
    }
    if (!*abort && i0 + tid < A.K)
      A.part[(int64_t)blockIdx.x * A.K + i0 + tid] =
          WHICH == 0 ? -fmaf(-gb_s, acc0, acc1) / (1.0f + acc0) : -acc1;
    ptx::tc_fence_before();
    __syncthreads();  // every epilogue of the round is done before the next round's noise
    ptx::tc_fence_after();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTcTmemCols);
}

// Value noise, step 1: w_s = sum_{t >= s} a_t,s e_t per head, the transpose
// of the clean pass. One CTA per (sequence, head, block of kFwdWarps key
// positions), one warp per key position s; the CTA's later query and error
// rows are staged through shared-memory tiles (row stride d_h + 4), and each
// warp forms a_t,s = exp(q_t . k_s c - LSE_t) for its tile rows, then adds
// a e_t into the lanes' d_h / 32 columns. Shared memory: kTile x (d_h + 4)
// for Q and for E, kTile LSE values, and per warp k_s (d_h) and the tile's
// a (kTile).
template <int DH>
__global__ __launch_bounds__(kFwdWarps * 32) void k_attn_colsum(const __grid_constant__ FwdArgs A,
                                                               float* __restrict__ W) {
  extern __shared__ __align__(16) float csm[];
  constexpr int kStride = DH + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrb = (A.L + kFwdWarps - 1) / kFwdWarps;
  const int rb = blockIdx.x % nrb;
  const int h = (blockIdx.x / nrb) % A.H;
  const int64_t seq = blockIdx.x / ((int64_t)nrb * A.H);
  const int64_t D = (int64_t)A.H * DH;
  const int64_t s0 = seq * A.L;
  const int pos = rb * kFwdWarps + warp;  // this warp's key position
  const bool ok = pos < A.L;
  const int first = rb * kFwdWarps;       // earliest query row any warp needs
  float* qt = csm;
  float* et = qt + kTile * kStride;
  float* lt = et + kTile * kStride;
  float* ks = lt + kTile + (size_t)warp * (DH + kTile);
  float* ab = ks + DH;
  if (ok)
    for (int c = lane; c < DH; c += 32) ks[c] = A.Kc[(s0 + pos) * D + h * DH + c];
  float w[DH / 32];
#pragma unroll
  for (int u = 0; u < DH / 32; ++u) w[u] = 0.f;
  for (int j0 = first; j0 < A.L; j0 += kTile) {
    const int rows = min(kTile, A.L - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < rows * (DH / 4); e += kFwdWarps * 32) {
      const int r = e / (DH / 4), c4 = e % (DH / 4);
      const int64_t src = (s0 + j0 + r) * D + h * DH;
      *reinterpret_cast<float4*>(qt + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.Q + src)[c4];
      *reinterpret_cast<float4*>(et + r * kStride + 4 * c4) =
          reinterpret_cast<const float4*>(A.E + src)[c4];
    }
    for (int r = threadIdx.x; r < rows; r += kFwdWarps * 32) lt[r] = A.lse[(s0 + j0 + r) * A.H + h];
    __syncthreads();
    if (ok) {
      for (int j = lane; j < rows; j += 32)
        ab[j] = (j0 + j >= pos) ? expf(dot_row<DH>(ks, qt + j * kStride) * A.scale - lt[j]) : 0.0f;
      __syncwarp();
      for (int j = 0; j < rows; ++j) {
        const float a = ab[j];
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) w[u] = fmaf(a, et[j * kStride + lane + 32 * u], w[u]);
      }
    }
  }
  if (!ok) return;  // after the last block barrier
#pragma unroll
  for (int u = 0; u < DH / 32; ++u) W[(s0 + pos) * D + h * DH + lane + 32 * u] = w[u];
}

// Value noise, step 2: r_s,i = -(sigma eps_s,i) . w_s over all D channels.
// One CTA per token, one thread per draw; the table carries sigma, so the
// Gaussians come out as sigma eps. Each counter (slot block, lane) gives the
// four channels blk 128 + lane + 32 j.
__global__ __launch_bounds__(kDrawThreads) void k_attn_vdraws(
    const float* __restrict__ W, int64_t D, RoundKeys keys, uint32_t t_off, uint32_t i_off,
    uint32_t ctr3, float sigma, int32_t K, float* __restrict__ r) {
  extern __shared__ __align__(16) float ws[];  // D, padded to 128
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, sigma);
  const int64_t s = blockIdx.x;
  const int nblk = (int)((D + 127) / 128);
  for (int c = threadIdx.x; c < nblk * 128; c += kDrawThreads) ws[c] = c < D ? W[s * D + c] : 0.f;
  __syncthreads();
  const uint32_t t_abs = t_off + (uint32_t)s;
  for (int i = threadIdx.x; i < K; i += kDrawThreads) {
    const DrawConst dc = draw_const(keys, t_abs, i_off + (uint32_t)i);
    float a0 = 0.f, a1 = 0.f;
    for (int blk = 0; blk < nblk; ++blk) {
      const float* wb = ws + blk * 128;
#pragma unroll 4
      for (int l = 0; l < 32; ++l) {
        const G4 g = gauss4_tab(
            philox_from2(block_const(keys, slot_ctr0((uint32_t)blk, (uint32_t)l), ctr3), dc, keys),
            tab);
        a0 = fmaf(g.v[0], wb[l], a0);
        a1 = fmaf(g.v[1], wb[l + 32], a1);
        a0 = fmaf(g.v[2], wb[l + 64], a0);
        a1 = fmaf(g.v[3], wb[l + 96], a1);
      }
    }
    r[s * K + i] = -(a0 + a1);
  }
}

// r[s K + i] = sum_h part[(s H + h) K + i], heads in order.
__global__ void k_attn_combine(const float* __restrict__ part, int64_t T, int32_t H, int32_t K,
                               float* __restrict__ r) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= T * K) return;
  const int64_t s = gid / K;
  const int32_t i = (int32_t)(gid % K);
  float acc = 0.f;
  for (int h = 0; h < H; ++h) acc += part[(s * H + h) * K + i];
  r[gid] = acc;
}

template <int DH>
cudaError_t fwd_dh(cudaStream_t st, const FwdArgs& A) {
  const bool kc = A.kcoef != nullptr;
  const size_t smem = attn_fwd_smem(A.L, DH, kc);
  auto fn = kc ? k_attn_fwd_kc<DH> : k_attn_fwd<DH>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t nrb = (A.L + kFwdWarps - 1) / kFwdWarps;
  const int64_t blocks = (A.T / A.L) * A.H * nrb;
  fn<<<(unsigned)blocks, kFwdWarps * 32, smem, st>>>(A);
  return cudaGetLastError();
}

template <int WHICH, int DH>
cudaError_t draws_dh(cudaStream_t st, const DrawArgs& A) {
  const size_t smem = attn_draws_smem(A.L, DH);
  cudaError_t e = cudaFuncSetAttribute(k_attn_draws<WHICH, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_attn_draws<WHICH, DH><<<(unsigned)(A.T * A.H), kDrawThreads, smem, st>>>(A);
  return cudaGetLastError();
}

template <int DH>
cudaError_t draws_which(cudaStream_t st, int which, const DrawArgs& A) {
  if (which == 0) return draws_dh<0, DH>(st, A);
  return draws_dh<1, DH>(st, A);
}

template <int DH>
cudaError_t kcoef_dh(cudaStream_t st, const FwdArgs& F, float2* C, size_t smem, unsigned blocks) {
  cudaError_t e = cudaFuncSetAttribute(k_attn_kcoef<DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_attn_kcoef<DH><<<blocks, kFwdWarps * 32, smem, st>>>(F, C);
  return cudaGetLastError();
}

template <int WHICH, int DH>
cudaError_t draws_tc(cudaStream_t st, const TcDrawArgs& A) {
  const size_t smem = attn_tc_smem(A.L, DH);
  cudaError_t e = cudaFuncSetAttribute(k_attn_draws_tc<WHICH, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_attn_draws_tc<WHICH, DH><<<(unsigned)(A.T * A.H), kDrawThreads, smem, st>>>(A);
  return cudaGetLastError();
}

template <int DH>
cudaError_t colsum_dh(cudaStream_t st, const FwdArgs& A, float* W) {
  const size_t smem = attn_colsum_smem(DH);
  cudaError_t e = cudaFuncSetAttribute(k_attn_colsum<DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t nrb = (A.L + kFwdWarps - 1) / kFwdWarps;
  k_attn_colsum<DH><<<(unsigned)((A.T / A.L) * A.H * nrb), kFwdWarps * 32, smem, st>>>(A, W);
  return cudaGetLastError();
}

}  // namespace

size_t attn_fwd_smem(int L, int head_dim, bool kcoef) {
  const size_t Lp = (size_t)((L + 3) & ~3);
  return ((size_t)kFwdWarps * (Lp + 2 * head_dim) + (size_t)kTile * (head_dim + 4) +
          (kcoef ? (size_t)kFwdWarps * (Lp + 1) : 0)) * 4;
}
size_t attn_coef_smem(int head_dim) {
  return ((size_t)2 * kTile * (head_dim + 4) + 2 * kTile + (size_t)kFwdWarps * 2 * head_dim) * 4;
}
size_t attn_tc_smem(int L, int head_dim) {
  const size_t kb = (size_t)head_dim / 64;
  return 1024 + 2 * 2 * kb * 128 * 128 + 2 * 2 * kb * kTcRows * 128 +
         (size_t)((L + kTcRows - 1) / kTcRows) * kTcRows * 8;
}
size_t attn_colsum_smem(int head_dim) {
  return ((size_t)2 * kTile * (head_dim + 4) + kTile + (size_t)kFwdWarps * (head_dim + kTile)) * 4;
}
size_t attn_draws_smem(int L, int head_dim) {
  return (size_t)(2 * ((L + 3) & ~3) + kTile * (head_dim + 8) + kDrawThreads * (head_dim + 1)) * 4;
}

cudaError_t launch_attn_fwd(cudaStream_t st, int64_t T, int L, int H, int head_dim,
                            const float* Q, const float* Kc, const float* Vc, const float* E,
                            float* O, float* lse, float* gbar, float2* qcoef, float2* kcoef) {
  FwdArgs A{Q, Kc, Vc, E, O, lse, gbar, T, L, H, 1.0f / sqrtf((float)head_dim), qcoef, kcoef};
  if (head_dim == 32) return fwd_dh<32>(st, A);
  if (head_dim == 64) return fwd_dh<64>(st, A);
  return fwd_dh<128>(st, A);
}

cudaError_t launch_attn_draws(cudaStream_t st, const dust_params& p, int which, int L, int H,
                              int head_dim, const float* Q, const float* Kc, const float* Vc,
                              const float* E, const float* O, const float* lse,
                              const float* gbar, float* part, float* W, float* r, bool use_tc,
                              uint8_t* tc_rows, float2* coef, bool coef_done, uint32_t* status) {
  if (p.T * H <= 0) return cudaSuccess;
  const float c = 1.0f / sqrtf((float)head_dim);
  const uint32_t ctr3 = ctr3_of(kTagAttnQ + which, p.stream_id);
  if (which == 2) {
    // value noise: w_s once, then one D-long dot per draw (rewards go to r)
    FwdArgs F{Q, Kc, Vc, E, nullptr, const_cast<float*>(lse), nullptr, p.T, L, H, c, nullptr};
    cudaError_t e = head_dim == 32 ? colsum_dh<32>(st, F, W)
                    : head_dim == 64 ? colsum_dh<64>(st, F, W) : colsum_dh<128>(st, F, W);
    if (e != cudaSuccess) return e;
    const int64_t D = (int64_t)H * head_dim;
    const size_t smem = (size_t)((D + 127) / 128) * 128 * 4;
    e = cudaFuncSetAttribute(k_attn_vdraws, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_attn_vdraws<<<(unsigned)p.T, kDrawThreads, smem, st>>>(
        W, D, round_keys(p.seed), (uint32_t)p.token_offset, (uint32_t)p.draw_offset, ctr3,
        p.sigma, p.K, r);
    return cudaGetLastError();
  }
  if (use_tc && head_dim >= 64) {
    // the noise's power-of-two factor S puts max |S sigma c eps| near 8
    float S = 1.0f;
    const float xmax = p.sigma * c * 5.7687f;
    if (xmax > 0.0f) S = exp2f(floorf(log2f(8.0f / xmax)));
    S = fminf(fmaxf(S, 0x1p-40f), 0x1p40f);
    const int ntile = (L + kTcRows - 1) / kTcRows;
    const unsigned units = (unsigned)((p.T / L) * H * ntile);
    const float* rsrc = which == 0 ? Kc : Q;
    if (head_dim == 64)
      k_attn_tc_rows<64><<<units, kDrawThreads, 0, st>>>(rsrc, p.T, L, H, tc_rows, status);
    else
      k_attn_tc_rows<128><<<units, kDrawThreads, 0, st>>>(rsrc, p.T, L, H, tc_rows, status);
    {
      FwdArgs F{Q, Kc, Vc, E, nullptr, const_cast<float*>(lse), const_cast<float*>(gbar), p.T, L,
                H, c, nullptr};
      const size_t csm = attn_coef_smem(head_dim);
      const unsigned cblocks = (unsigned)((p.T / L) * H * ((L + kFwdWarps - 1) / kFwdWarps));
      // query noise, and key noise where the rows fit its shared memory: the
      // clean pass wrote the rows (launch_attn_fwd's qcoef, kcoef)
      cudaError_t ce = cudaSuccess;
      if (which == 1 && !coef_done)
        ce = head_dim == 64 ? kcoef_dh<64>(st, F, coef, csm, cblocks)
                            : kcoef_dh<128>(st, F, coef, csm, cblocks);
      if (ce != cudaSuccess) return ce;
    }
    TcDrawArgs T{gbar, part, tc_rows, coef, round_keys(p.seed), (uint32_t)p.token_offset,
                 (uint32_t)p.draw_offset, ctr3, p.sigma * c * S, 1.0f / S, p.T, L, H, p.K,
                 status};
    cudaError_t e = head_dim == 64 ? (which == 0 ? draws_tc<0, 64>(st, T) : draws_tc<1, 64>(st, T))
                                   : (which == 0 ? draws_tc<0, 128>(st, T) : draws_tc<1, 128>(st, T));
    if (e != cudaSuccess) return e;
    return launch_attn_combine(st, part, p.T, H, p.K, r);
  }
  DrawArgs A{Q, Kc, Vc, E, O, lse, gbar, part, round_keys(p.seed), (uint32_t)p.token_offset,
             (uint32_t)p.draw_offset, ctr3, p.sigma * c, p.T, L, H, p.K, c};
  cudaError_t e = head_dim == 32 ? draws_which<32>(st, which, A)
                  : head_dim == 64 ? draws_which<64>(st, which, A) : draws_which<128>(st, which, A);
  if (e != cudaSuccess) return e;
  return launch_attn_combine(st, part, p.T, H, p.K, r);
}

cudaError_t launch_attn_combine(cudaStream_t st, const float* part, int64_t T, int H, int K,
                                float* r) {
  const int64_t n = T * K;
  if (n <= 0) return cudaSuccess;
  k_attn_combine<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, T, H, K, r);
  return cudaGetLastError();
}

}  // namespace dust

namespace dust {
size_t attn_tc_rows_bytes(int64_t T, int L, int H, int head_dim) {
  const int64_t ntile = (L + kTcRows - 1) / kTcRows;
  return (size_t)(T / L) * H * ntile * 2 * (head_dim / 64) * kTcRows * 128;
}
size_t attn_coef_bytes(int64_t T, int L, int H) {
  return (size_t)T * H * ((L + kTcRows - 1) / kTcRows * kTcRows) * 8;
}
}  // namespace dust
