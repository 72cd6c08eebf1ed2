// Full-vocabulary LM-head draws ("Dust：无需反向传播的Transformer零阶预训练",
// §1): every logit of token t gets sigma*eps; the perturbed loss is formed in
// delta form from the softmax p = exp(z - LSE) of the cached clean logits,
//   L' - L = log1p(sum_j p_j expm1(sigma eps_j)) - sigma eps_y,
// the reward is r = L - L', and g_t = -(1/(K sigma)) sum_i r_i eps_i.
// The reward needs the whole row before any g entry can be formed. The
// one-pass kernel (k_full_one, below) keeps a token's row and two draws of its
// noise in the shared memory of a cluster and exchanges each draw's row sum
// across the cluster; where no cluster configuration fits, the noise is
// generated twice (stage 1 and stage 3). It never reaches global memory.
//
// Both noise passes are persistent over (token, 3072-entry slab) units: a warp
// owns three 128-slot blocks of the slab, evaluates Philox rounds 0-1 of its
// blocks once per unit and those of each draw once per draw, and turns words
// into sigma-scaled Gaussians with the table-driven Box-Muller step (the
// table of roots of unity is built once per CTA). Stage 1 also records the
// target's noise, so stage 2 needs none of its own.
#include "internal.cuh"
#include "noise.cuh"
#include "tc_ptx.cuh"

#include <cmath>
#include <cstdint>
#include <mutex>

namespace dust {
namespace {

constexpr int kWarps = 8;
// 128-slot blocks per warp: three keeps both passes within 64 registers, so
// they run 32 warps per SM (four blocks, 72 registers in the reward pass:
// 24 warps; 2 % slower on full_bf16)
constexpr int kBlocksPerWarp = 3;
constexpr int kSlab = kWarps * kBlocksPerWarp * 128;  // vocabulary entries per unit
constexpr int kDrawChunk = 64;
// The Box-Muller step in packed fp32x2 form (PACKED) or scalar and paired up
// afterwards. Packed operations run on the FMA-heavy pipe, which the Philox
// multiplies also need: measured on B200, the reward pass (with its packed
// expm1 and sums) is faster with the packed step (15.5 against 15.9 ms on
// full_bf16), the g pass with the scalar one (12.3 against 12.5 ms).
template <bool PACKED>
__device__ __forceinline__ void noise4(U4 w, const float2* tab, float2& e02, float2& e13) {
  if (PACKED) {
    gauss4_tab_x2(w, tab, e02, e13);
  } else {
    const G4 g = gauss4_tab(w, tab);
    e02 = make_float2(g.v[0], g.v[2]);
    e13 = make_float2(g.v[1], g.v[3]);
  }
}

struct FullArgs {
  RoundKeys keys;
  uint32_t t_off, i_off, ctr3;
  float sigma;
  float fac;  // g = fac * sum_i r_i (sigma eps_i)
  int64_t T, V;
  int32_t K;
  int nslab;
  const float* Z;    // clean logits (T x V)
  const float* lse;  // T
  const int32_t* y;
  float* part;       // (t * nslab + slab) * K + i
  float* xy;         // sigma eps at the target, t * K + i
  const float* r;    // rewards, t * K + i
  float* g_out;
  void* gop;
  GopFormat gf;
  int64_t plane;
  // one pass
  float* r_out;       // rewards t * K + i (may be null)
  uint32_t* status;   // kStatusTimeout
  int32_t nb, bpc;    // CTAs per cluster, 128-slot blocks per CTA
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Draws [i0, i0 + n) of one unit for one warp; per draw, the warp's sum goes
// to sh[warp][ii]. ALL: all kBlocksPerWarp blocks of the warp lie below V
// (every warp but the one that straddles V), so no per-block test runs in the
// draw loop. The noise, expm1 and the reward sums run in packed fp32x2
// arithmetic on the pairs of slots (lane, lane + 64) and (lane + 32, lane + 96)
// of each block (p02, p13), one pair of chains per block. No barrier inside:
// the caller's block-wide barriers are the same for every warp.
template <int DEG, bool ALL>
__device__ __forceinline__ void reward_chunk(const FullArgs& A, const float2* tab, int64_t t,
                                             int i0, int n, int nvalid,
                                             const float2 (&p02)[kBlocksPerWarp],
                                             const float2 (&p13)[kBlocksPerWarp],
                                             const BlockConst (&bc)[kBlocksPerWarp],
                                             bool warp_has_y, bool y_here, int by, int jy,
                                             float (*sh)[kDrawChunk]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t t_abs = A.t_off + (uint32_t)t;
  for (int ii = 0; ii < n; ++ii) {
    const uint32_t i_abs = A.i_off + (uint32_t)(i0 + ii);
    const DrawConst dc = draw_const(A.keys, t_abs, i_abs);
    float sb[kBlocksPerWarp];
    float xyv = 0.0f;
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      sb[b] = 0.0f;
      if (ALL || b < nvalid) {
        float2 e02, e13;
        noise4<true>(philox_from2(bc[b], dc, A.keys), tab, e02, e13);
        float2 s2 = __fmul2_rn(p02[b], expm1_small_x2<DEG>(e02));
        s2 = __ffma2_rn(p13[b], expm1_small_x2<DEG>(e13), s2);
        sb[b] = s2.x + s2.y;
        if (warp_has_y && b == by) {
          // word jy of the counter: 0, 2 in e02 and 1, 3 in e13
          const float2 e = (jy & 1) ? e13 : e02;
          xyv = (jy & 2) ? e.y : e.x;
        }
      }
    }
    if (y_here) A.xy[t * A.K + i0 + ii] = xyv;
    float s = 0.0f;
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) s += sb[b];
    s = warp_sum(s);
    if (lane == 0) sh[warp][ii] = s;
  }
}

template <int DEG>
__global__ __launch_bounds__(kWarps * 32) void k_full_reward_partial(const __grid_constant__ FullArgs A) {
  __shared__ float sh[kWarps][kDrawChunk];
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, A.sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nunits = A.T * A.nslab;
  for (int64_t unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int64_t t = unit / A.nslab;
    const int slab = (int)(unit % A.nslab);
    const int64_t blk0 = (int64_t)slab * (kSlab / 128) + warp * kBlocksPerWarp;
    // blocks of this warp below V (warp-uniform)
    const int64_t left = (A.V - blk0 * 128 + 127) / 128;
    const int nvalid = left <= 0 ? 0 : (left >= kBlocksPerWarp ? kBlocksPerWarp : (int)left);
    // p = exp(z - LSE), formed once per unit, as the packed pairs of slots
    // (lane, lane + 64) and (lane + 32, lane + 96) of each block
    float2 p02[kBlocksPerWarp], p13[kBlocksPerWarp];
    BlockConst bc[kBlocksPerWarp];
    const float lse_t = A.lse[t];
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      bc[b] = block_const(A.keys, slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), A.ctr3);
      float pv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
        pv[j] = pos < A.V ? expf(A.Z[t * A.V + pos] - lse_t) : 0.0f;
      }
      p02[b] = make_float2(pv[0], pv[2]);
      p13[b] = make_float2(pv[1], pv[3]);
    }
    // the lane holding the target's noise, if this warp's blocks contain it
    int32_t yt = A.y[t];
    if (yt < 0 || (int64_t)yt >= A.V) yt = 0;  // reported by the loss kernel
    const int64_t yb = (int64_t)yt >> 7;
    const bool warp_has_y = yb >= blk0 && yb < blk0 + kBlocksPerWarp;  // warp-uniform
    const bool y_here = warp_has_y && lane == (yt & 31);
    const int by = (int)(yb - blk0), jy = (yt >> 5) & 3;
    for (int i0 = 0; i0 < A.K; i0 += kDrawChunk) {
      const int n = min(kDrawChunk, A.K - i0);
      if (nvalid == kBlocksPerWarp)
        reward_chunk<DEG, true>(A, tab, t, i0, n, nvalid, p02, p13, bc, warp_has_y, y_here, by, jy, sh);
      else
        reward_chunk<DEG, false>(A, tab, t, i0, n, nvalid, p02, p13, bc, warp_has_y, y_here, by, jy, sh);
      __syncthreads();
      if ((int)threadIdx.x < n) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += sh[w][threadIdx.x];
        A.part[(t * A.nslab + slab) * (int64_t)A.K + i0 + threadIdx.x] = s;
      }
      __syncthreads();
    }
  }
}

__global__ void k_full_reward_combine(int64_t T, int32_t K, int nslab,
                                      const float* __restrict__ part,
                                      const float* __restrict__ xy, float* __restrict__ r) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= T * K) return;
  const int64_t t = id / K;
  const int32_t i = (int32_t)(id % K);
  float s = 0.0f;
  for (int sl = 0; sl < nslab; ++sl) s += part[(t * nslab + sl) * (int64_t)K + i];
  r[id] = xy[id] - log1pf(s);
}

// Draws [i0, i0 + n) of sum_i r_i (sigma eps_i) for one warp's blocks, with
// r staged in rs (ALL: every block lies below V), accumulated in packed pairs
// (slots lane, lane + 64 in acc02; lane + 32, lane + 96 in acc13). No barrier
// inside.
template <bool ALL>
__device__ __forceinline__ void g_chunk(const FullArgs& A, const float2* tab, int64_t t, int i0,
                                        int n, int nvalid, const BlockConst (&bc)[kBlocksPerWarp],
                                        const float* rs, float2 (&acc02)[kBlocksPerWarp],
                                        float2 (&acc13)[kBlocksPerWarp]) {
  const uint32_t t_abs = A.t_off + (uint32_t)t;
  for (int ii = 0; ii < n; ++ii) {
    const float ri = rs[ii];
    const float2 r2 = make_float2(ri, ri);
    const DrawConst dc = draw_const(A.keys, t_abs, A.i_off + (uint32_t)(i0 + ii));
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      if (ALL || b < nvalid) {
        float2 e02, e13;
        noise4<false>(philox_from2(bc[b], dc, A.keys), tab, e02, e13);
        acc02[b] = __ffma2_rn(r2, e02, acc02[b]);
        acc13[b] = __ffma2_rn(r2, e13, acc13[b]);
      }
    }
  }
}

__global__ __launch_bounds__(kWarps * 32) void k_full_g(const __grid_constant__ FullArgs A) {
  __shared__ float rs[1024];
  __shared__ float2 tab[kSinCosTable];
  fill_sincos_table(tab, A.sigma);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nunits = A.T * A.nslab;
  for (int64_t unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    const int64_t t = unit / A.nslab;
    const int slab = (int)(unit % A.nslab);
    const int64_t blk0 = (int64_t)slab * (kSlab / 128) + warp * kBlocksPerWarp;
    const int64_t left = (A.V - blk0 * 128 + 127) / 128;
    const int nvalid = left <= 0 ? 0 : (left >= kBlocksPerWarp ? kBlocksPerWarp : (int)left);
    BlockConst bc[kBlocksPerWarp];
    float2 acc02[kBlocksPerWarp], acc13[kBlocksPerWarp];
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      bc[b] = block_const(A.keys, slot_ctr0((uint32_t)(blk0 + b), (uint32_t)lane), A.ctr3);
      acc02[b] = make_float2(0.0f, 0.0f);
      acc13[b] = make_float2(0.0f, 0.0f);
    }
    for (int i0 = 0; i0 < A.K; i0 += 1024) {
      const int n = min(1024, A.K - i0);
      __syncthreads();
      for (int q = threadIdx.x; q < n; q += blockDim.x) rs[q] = A.r[t * A.K + i0 + q];
      __syncthreads();
      if (nvalid == kBlocksPerWarp)
        g_chunk<true>(A, tab, t, i0, n, nvalid, bc, rs, acc02, acc13);
      else
        g_chunk<false>(A, tab, t, i0, n, nvalid, bc, rs, acc02, acc13);
    }
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t pos = (blk0 + b) * 128 + lane + 32 * j;
        if (pos < A.V) {
          const float2 a = (j & 1) ? acc13[b] : acc02[b];
          const float v = ((j & 2) ? a.y : a.x) * A.fac;
          if (A.g_out) A.g_out[t * A.V + pos] = v;
          store_gop(A.gop, A.gf, A.plane, t * A.V + pos, v);
        }
      }
  }
}

// ---- one pass: the noise generated once -------------------------------------
// A cluster of nb CTAs owns one token's row at a time: CTA c holds the 128-slot
// blocks [c * bpc, (c + 1) * bpc), with p = exp(z - LSE), the g accumulators and
// two buffers of noise in shared memory (the four slots of a lane side by side,
// in the order 0, 2, 1, 3 of the packed pairs). Warps 0..W-1 generate: warp w
// takes the blocks w, w + W, w + 2W, ... (at most kOneR) of its CTA. For draw i it writes the
// blocks' sigma*eps to buffer i & 1, adds up p * expm1(sigma eps), and posts the
// warp's sum to its CTA's reducer (shared memory, then an arrive on the draw's
// local barrier); it then takes the reward of draw i - 1 from the reducer and
// adds r * sigma eps of buffer (i - 1) & 1 to its accumulators, so the exchange
// of a draw overlaps the generation of the next. Warp W reduces: it sums the
// warps' shares of a draw, sends the CTA's total to every CTA of the cluster
// (st.async, completing bytes on the receiver's barrier of the draw), forms
// r = sigma eps_y - log1p(sum of the totals) once all have arrived (sigma eps_y
// from the target's counter, evaluated by the reducer itself, 32 draws per
// lane at a time), and posts it on the local barrier the generators wait on.
// Four slots per barrier: a generator posts draw k + 4 only after it has read
// the reward of draw k + 3, which the reducer posts only after the totals of
// draw k + 3 arrived from every CTA, each sent after that CTA's reducer had
// read its totals of draw k + 2; so no slot is rewritten while still read, and
// no barrier runs a phase ahead of a waiting warp. Every wait is bounded (2 s,
// then the status word's timeout bit and no further waits).
constexpr int kOneSlots = 4;
constexpr int kOneMaxW = 31;  // generator warps (one more reduces)
// blocks per generator warp: 5 measured best on full_bf16 (23.1 ms against 24.7
// at 4, 26.5 at 6, 25.8 at 7; clusters of 4, so 20, 25, 17 and 15 warps)
constexpr int kOneR = 5;
constexpr int kOneOffL = kSinCosTable * 8;             // warp shares [4][32]
constexpr int kOneOffC = kOneOffL + kOneSlots * 32 * 4;  // CTA totals [4][8]
constexpr int kOneOffR = kOneOffC + kOneSlots * 8 * 4;   // rewards [4]
constexpr int kOneOffBar = kOneOffR + kOneSlots * 4 + 16;
constexpr int kOneOffP = (kOneOffBar + 3 * kOneSlots * 8 + 15) / 16 * 16;

__host__ __device__ constexpr size_t one_smem_bytes(int bpc) {
  return (size_t)kOneOffP + (size_t)bpc * 4 * 512;  // p, g and two noise buffers
}

__device__ __forceinline__ void one_st_async(uint32_t addr, float x, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(addr),
               "f"(x), "r"(remote_bar)
               : "memory");
}
__device__ __forceinline__ bool one_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void one_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void one_wait(uint32_t bar, uint32_t parity, uint32_t* status, bool& dead) {
  if (dead || one_try_wait(bar, parity)) return;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (one_try_wait(bar, parity)) return;
    if ((it & 63u) == 0 && ptx::globaltimer_ns() - t0 > 2000000000ull) {
      atomicOr(status, kStatusTimeout);
      dead = true;
      return;
    }
  }
}
// component of slot q (0..3 of a lane's counter) in the (0, 2, 1, 3) order
__device__ __forceinline__ int one_comp(int q) { return (q & 1) ? 2 + (q >> 1) : (q >> 1); }

template <int DEG>
__global__ __launch_bounds__((kOneMaxW + 1) * 32, 1) void k_full_one(const __grid_constant__ FullArgs A) {
  extern __shared__ __align__(16) uint8_t one_smem[];
  float2* tab = (float2*)one_smem;
  float* lpart = (float*)(one_smem + kOneOffL);
  float* cpart = (float*)(one_smem + kOneOffC);
  float* rs = (float*)(one_smem + kOneOffR);
  uint64_t* Lb = (uint64_t*)(one_smem + kOneOffBar);  // warp shares in (W arrivals)
  uint64_t* Cb = Lb + kOneSlots;                       // CTA totals in (bytes)
  uint64_t* Rb = Cb + kOneSlots;                       // reward out (1 arrival)
  float4* p4 = (float4*)(one_smem + kOneOffP);
  float4* g4 = p4 + (size_t)A.bpc * 32;
  float4* e4 = g4 + (size_t)A.bpc * 32;  // two buffers of bpc * 32
  const int nb = A.nb;
  const uint32_t rank = ptx::cluster_ctarank();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = (int)(blockDim.x >> 5) - 1;
  const bool reducer = warp == W;
  fill_sincos_table(tab, A.sigma);
  const int64_t nblocks = (A.V + 127) >> 7;
  const int64_t cb0 = (int64_t)rank * A.bpc;
  const int64_t left = nblocks - cb0;
  const int nloc = left <= 0 ? 0 : (left < A.bpc ? (int)left : A.bpc);
  if (threadIdx.x == 0) {
    for (int q = 0; q < kOneSlots; ++q) {
      ptx::mbar_init(ptx::smem_u32(&Lb[q]), (uint32_t)W);
      ptx::mbar_init(ptx::smem_u32(&Cb[q]), 1u);
      ptx::mbar_init(ptx::smem_u32(&Rb[q]), 1u);
    }
    ptx::fence_barrier_init();
    for (int q = 0; q < kOneSlots; ++q) ptx::mbar_expect_tx(ptx::smem_u32(&Cb[q]), (uint32_t)(nb * 4));
  }
  __syncthreads();
  ptx::cluster_sync();  // every CTA's barriers exist before the first remote store
  const int nmine = (!reducer && warp < nloc) ? min(kOneR, (nloc - 1 - warp) / W + 1) : 0;
  BlockConst bc[kOneR];
#pragma unroll
  for (int j = 0; j < kOneR; ++j)
    bc[j] = block_const(A.keys, slot_ctr0((uint32_t)(cb0 + warp + W * j), (uint32_t)lane), A.ctr3);
  const int64_t ncl = gridDim.x / nb, cid = blockIdx.x / nb;
  const int nslots = nloc * 128;
  uint32_t kg = 0;  // draws this cluster has run: the slot and phase of a draw
  bool dead = false;
  for (int64_t t = cid; t < A.T; t += ncl) {
    __syncthreads();  // the previous token's g is written out
    const float lse_t = A.lse[t];
    const float* zrow = A.Z + t * A.V + (cb0 << 7);
    const int64_t vrem = A.V - (cb0 << 7);  // slots of this CTA below V
    for (int base = 0; base < nslots; base += 4 * (int)blockDim.x) {
      float zv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = base + u * (int)blockDim.x + (int)threadIdx.x;
        zv[u] = idx < vrem && idx < nslots ? zrow[idx] : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = base + u * (int)blockDim.x + (int)threadIdx.x;
        if (idx < nslots) {
          const int o = ((idx >> 7) * 32 + (idx & 31)) * 4 + one_comp((idx >> 5) & 3);
          ((float*)p4)[o] = idx < vrem ? expf(zv[u] - lse_t) : 0.0f;
          ((float*)g4)[o] = 0.0f;
        }
      }
    }
    int32_t yt = A.y[t];
    if (yt < 0 || (int64_t)yt >= A.V) yt = 0;  // reported by the loss kernel
    __syncthreads();
    const uint32_t t_abs = A.t_off + (uint32_t)t;
    const int K = A.K;
    if (reducer) {
      const BlockConst bcy =
          block_const(A.keys, slot_ctr0((uint32_t)(yt >> 7), (uint32_t)(yt & 31)), A.ctr3);
      const int qy = (yt >> 5) & 3;
      float ycur = 0.0f;
      for (int i = 0; i < K; ++i) {
        const uint32_t k = kg + (uint32_t)i, slot = k % kOneSlots, par = (k / kOneSlots) & 1u;
        if ((i & 31) == 0) {  // sigma eps at the target for draws i .. i + 31, one per lane
          float2 a, b;
          noise4<true>(philox_from2(bcy, draw_const(A.keys, t_abs, A.i_off + (uint32_t)(i + lane)),
                                    A.keys),
                       tab, a, b);
          const float lo = (qy & 1) ? b.x : a.x, hi = (qy & 1) ? b.y : a.y;
          ycur = (qy & 2) ? hi : lo;
        }
        one_wait(ptx::smem_u32(&Lb[slot]), par, A.status, dead);
        float s = 0.0f;
        for (int q = lane; q < W; q += 32) s += lpart[slot * 32 + q];
        s = warp_sum(s);
        if (lane < nb)
          one_st_async(ptx::mapa_shared(ptx::smem_u32(&cpart[slot * 8 + rank]), (uint32_t)lane), s,
                       ptx::mapa_shared(ptx::smem_u32(&Cb[slot]), (uint32_t)lane));
        one_wait(ptx::smem_u32(&Cb[slot]), par, A.status, dead);
        float S = 0.0f;
        for (int q = 0; q < nb; ++q) S += cpart[slot * 8 + q];
        // the slot's next use (draw k + 4) expects the totals again
        if (lane == 0) ptx::mbar_expect_tx(ptx::smem_u32(&Cb[slot]), (uint32_t)(nb * 4));
        const float r = __shfl_sync(0xffffffffu, ycur, i & 31) - log1pf(S);
        if (lane == 0) {
          if (A.r_out && rank == 0) A.r_out[t * K + i] = r;
          rs[slot] = r;
          one_arrive(ptx::smem_u32(&Rb[slot]));
        }
        __syncwarp();
      }
    } else {
      for (int i = 0; i <= K; ++i) {
        if (i < K) {  // generate draw i and post this warp's share
          const DrawConst dc = draw_const(A.keys, t_abs, A.i_off + (uint32_t)i);
          float2 acc = make_float2(0.0f, 0.0f);
          float4* eb = e4 + (size_t)(i & 1) * A.bpc * 32;
#pragma unroll
          for (int j = 0; j < kOneR; ++j) {
            if (j < nmine) {
              const int o = (warp + W * j) * 32 + lane;
              // the scalar Box-Muller step: its operations spread over both FMA
              // pipes, where the packed form loads the FMA-heavy one the Philox
              // multiplies already keep busy (0.7 % faster here)
              float2 e02, e13;
              noise4<false>(philox_from2(bc[j], dc, A.keys), tab, e02, e13);
              const float4 pv = p4[o];
              eb[o] = make_float4(e02.x, e02.y, e13.x, e13.y);
              acc = __ffma2_rn(make_float2(pv.x, pv.y), expm1_small_x2<DEG>(e02), acc);
              acc = __ffma2_rn(make_float2(pv.z, pv.w), expm1_small_x2<DEG>(e13), acc);
            }
          }
          const float s = warp_sum(acc.x + acc.y);
          const uint32_t slot = (kg + (uint32_t)i) % kOneSlots;
          if (lane == 0) {
            lpart[slot * 32 + warp] = s;
            one_arrive(ptx::smem_u32(&Lb[slot]));
          }
        }
        if (i > 0) {  // the reward of draw i - 1 into the accumulators
          const uint32_t k = kg + (uint32_t)(i - 1), slot = k % kOneSlots, par = (k / kOneSlots) & 1u;
          one_wait(ptx::smem_u32(&Rb[slot]), par, A.status, dead);
          const float r = rs[slot];
          const float2 r2 = make_float2(r, r);
          const float4* eb = e4 + (size_t)((i - 1) & 1) * A.bpc * 32;
#pragma unroll
          for (int j = 0; j < kOneR; ++j) {
            if (j < nmine) {
              const int o = (warp + W * j) * 32 + lane;
              const float4 e = eb[o];
              const float4 g = g4[o];
              const float2 lo = __ffma2_rn(r2, make_float2(e.x, e.y), make_float2(g.x, g.y));
              const float2 hi = __ffma2_rn(r2, make_float2(e.z, e.w), make_float2(g.z, g.w));
              g4[o] = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
          }
        }
      }
    }
    kg += (uint32_t)K;
    __syncthreads();
    for (int idx = threadIdx.x; idx < nslots; idx += blockDim.x) {
      if (idx < vrem) {
        const int o = ((idx >> 7) * 32 + (idx & 31)) * 4 + one_comp((idx >> 5) & 3);
        const float v = ((const float*)g4)[o] * A.fac;
        const int64_t off = t * A.V + (cb0 << 7) + idx;
        if (A.g_out) A.g_out[off] = v;
        store_gop(A.gop, A.gf, A.plane, off, v);
      }
    }
  }
  // every warp has seen every draw's exchange complete: no CTA addresses a peer
  // any more; none leaves before all are done
  ptx::cluster_sync();
}

FullArgs make_args(const dust_params& p) {
  FullArgs A{};
  A.keys = round_keys(p.seed);
  A.t_off = (uint32_t)p.token_offset;
  A.i_off = (uint32_t)p.draw_offset;
  A.ctr3 = ctr3_of(kTagHead, p.stream_id);
  A.sigma = p.sigma;
  const double s2 = (double)p.sigma * (double)p.sigma;
  A.fac = p.sigma > 0.0f ? (float)(-1.0 / ((double)p.K * s2)) : 0.0f;
  A.T = p.T;
  A.V = p.V;
  A.K = p.K;
  A.nslab = (int)((p.V + kSlab - 1) / kSlab);
  A.plane = p.T * p.V;
  return A;
}

// Persistent grid: every SM filled with as many CTAs as fit, at most one per unit;
// with `side`, side->sms SMs and CTAs of side->pad bytes of dynamic shared memory.
template <typename F>
int grid_for(F kernel, int64_t units, const FullSide* side = nullptr) {
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (side) sms = side->sms;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarps * 32,
                                                    side ? side->pad : 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cudaGetLastError();
  const int64_t g = (int64_t)sms * per_sm;
  return (int)(units < g ? units : g);
}

}  // namespace

int full_vocab_nslab(int64_t V) { return (int)((V + kSlab - 1) / kSlab); }

size_t full_vocab_xy_bytes(int64_t T, int32_t K) { return (size_t)T * K * 4; }

cudaError_t launch_full_reward_partial(cudaStream_t st, const dust_params& p, const float* Z,
                                       const float* lse, const int32_t* y, float* part,
                                       float* xy, const FullSide* side) {
  FullArgs A = make_args(p);
  A.Z = Z;
  A.lse = lse;
  A.y = y;
  A.part = part;
  A.xy = xy;
  const int64_t units = A.T * A.nslab;
  const size_t pad = side ? side->pad : 0;
  switch (expm1_degree(p.sigma)) {
    case 3:
      k_full_reward_partial<3><<<grid_for(k_full_reward_partial<3>, units, side), kWarps * 32, pad, st>>>(A);
      break;
    case 4:
      k_full_reward_partial<4><<<grid_for(k_full_reward_partial<4>, units, side), kWarps * 32, pad, st>>>(A);
      break;
    default:
      k_full_reward_partial<0><<<grid_for(k_full_reward_partial<0>, units, side), kWarps * 32, pad, st>>>(A);
  }
  return cudaGetLastError();
}

cudaError_t launch_full_reward_combine(cudaStream_t st, const dust_params& p, const float* part,
                                       const float* xy, float* r) {
  const int64_t n = p.T * (int64_t)p.K;
  const int threads = 256;
  k_full_reward_combine<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
      p.T, p.K, full_vocab_nslab(p.V), part, xy, r);
  return cudaGetLastError();
}

cudaError_t launch_full_g(cudaStream_t st, const dust_params& p, const float* r, float* g_out,
                          void* gop, GopFormat gf, const FullSide* side) {
  FullArgs A = make_args(p);
  A.r = r;
  A.g_out = g_out;
  A.gop = gop;
  A.gf = gf;
  k_full_g<<<grid_for(k_full_g, A.T * A.nslab, side), kWarps * 32, side ? side->pad : 0, st>>>(A);
  return cudaGetLastError();
}

// ---- one-pass plan and launch -----------------------------------------------
namespace {

using OneFn = void (*)(const FullArgs);

OneFn one_fn(int deg) {
  if (deg == 3) return k_full_one<3>;
  if (deg == 4) return k_full_one<4>;
  return k_full_one<0>;
}

cudaLaunchConfig_t one_cfg(cudaLaunchAttribute* attr, int nb, int W, size_t smem, int ncl,
                           cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)nb;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(ncl * nb));
  cfg.blockDim = dim3((unsigned)((W + 1) * 32));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

struct OnePlanEntry {
  int dev, deg, max_smem;
  int64_t V, T;
  FullOnePlan plan;
  bool ok;
};
std::mutex g_one_mu;
OnePlanEntry g_one_cache[16];
int g_one_n = 0;

}  // namespace

// Clusters of up to 4 CTAs (larger ones fit fewer SMs; measured slower): the one
// with the least work per SM, counting per draw W generator warps of kOneR
// block rounds each, and ceil(T / clusters) tokens per cluster, clusters beyond one
// per SM sharing their SMs.
bool full_one_plan(const dust_params& p, int sm_count, int max_smem_optin, FullOnePlan* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const int deg = expm1_degree(p.sigma);
  {
    std::lock_guard<std::mutex> lk(g_one_mu);
    for (int i = 0; i < g_one_n; ++i) {
      const OnePlanEntry& e = g_one_cache[i];
      if (e.dev == dev && e.deg == deg && e.max_smem == max_smem_optin && e.V == p.V && e.T == p.T) {
        *out = e.plan;
        return e.ok;
      }
    }
  }
  const int64_t nblocks = (p.V + 127) / 128;
  FullOnePlan best;
  double best_cost = 0.0;
  bool found = false;
  OneFn fn = one_fn(deg);
  for (int nb = 1; nb <= 4; ++nb) {
    const int64_t bpc = (nblocks + nb - 1) / nb;
    const size_t smem = one_smem_bytes((int)bpc);
    const int W = (int)((bpc + kOneR - 1) / kOneR);
    if (smem > (size_t)max_smem_optin || W < 1 || W > kOneMaxW) continue;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg =
        one_cfg(attr, nb, W, smem, sm_count / nb > 0 ? sm_count / nb : 1, 0);
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, (void*)fn, &cfg) != cudaSuccess || ncl < 1) {
      cudaGetLastError();
      continue;
    }
    const int64_t nc = ncl < p.T ? ncl : p.T;
    const double share = (double)(nc * nb) / (sm_count > 0 ? sm_count : 1);
    const double cost = (double)((p.T + nc - 1) / nc) * W * (share > 1.0 ? share : 1.0);
    if (!found || cost < best_cost) {
      found = true;
      best_cost = cost;
      best.nb = nb;
      best.W = W;
      best.ncl = (int)nc;
      best.smem = smem;
    }
  }
  {
    std::lock_guard<std::mutex> lk(g_one_mu);
    OnePlanEntry& e = g_one_cache[g_one_n < 16 ? g_one_n++ : (int)(p.V % 16)];
    e = OnePlanEntry{dev, deg, max_smem_optin, p.V, p.T, best, found};
  }
  *out = best;
  return found;
}

cudaError_t launch_full_one(cudaStream_t st, const dust_params& p, const FullOnePlan& plan,
                            const float* Z, const float* lse, const int32_t* y, float* r,
                            float* g_out, void* gop, GopFormat gf, uint32_t* status) {
  if (plan.nb < 1 || plan.W < 1 || plan.ncl < 1 || !status) return cudaErrorInvalidValue;
  FullArgs A = make_args(p);
  A.Z = Z;
  A.lse = lse;
  A.y = y;
  A.r_out = r;
  A.g_out = g_out;
  A.gop = gop;
  A.gf = gf;
  A.status = status;
  A.nb = plan.nb;
  A.bpc = (int32_t)((((p.V + 127) / 128) + plan.nb - 1) / plan.nb);
  OneFn fn = one_fn(expm1_degree(p.sigma));
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = one_cfg(attr, plan.nb, plan.W, plan.smem, plan.ncl, st);
  e = cudaLaunchKernelEx(&cfg, fn, A);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Per SM, the one-pass kernel finishes this many times the tokens of the two passes
// (4096 tokens of V = 50304, K = 64: 23.2 ms on 132 SMs against 14.9 + 12.4 ms on 148).
constexpr double kOneVsTwo = 1.3;

int64_t full_split_plan(const dust_params& p, const FullOnePlan& one, int sm_count,
                        FullSide* side) {
  const int used = one.nb * one.ncl;
  const int free_sms = sm_count - used;
  if (one.ncl < 1 || free_sms < 8) return 0;
  int dev = 0, cap = 0, res = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&cap, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&res, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  // the two passes' CTAs, padded, must not fit into what a one-pass CTA leaves of an SM
  const void* fns[2] = {(const void*)k_full_g, (const void*)k_full_reward_partial<0>};
  const int deg = expm1_degree(p.sigma);
  if (deg == 3) fns[1] = (const void*)k_full_reward_partial<3>;
  if (deg == 4) fns[1] = (const void*)k_full_reward_partial<4>;
  size_t stat = SIZE_MAX;
  for (const void* f : fns) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, f) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    if (fa.sharedSizeBytes < stat) stat = fa.sharedSizeBytes;
  }
  const int64_t left = (int64_t)cap - (int64_t)one.smem - 2 * (int64_t)res - (int64_t)stat;
  const size_t pad = left < 0 ? 0 : (size_t)((left + 128) / 128 * 128);
  if (pad > 48 * 1024) return 0;
  // the one-pass clusters take a whole number of rounds of tokens
  const double share1 = used * kOneVsTwo / (used * kOneVsTwo + free_sms);
  const int64_t rounds = (int64_t)std::llround((double)p.T * share1 / one.ncl);
  const int64_t T1 = rounds * one.ncl;
  if (rounds < 4 || T1 >= p.T) return 0;
  side->sms = free_sms;
  side->pad = pad;
  return p.T - T1;
}

}  // namespace dust
