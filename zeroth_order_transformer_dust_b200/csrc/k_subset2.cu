// Vocabulary-subset LM-head draws, shared-memory resident (the kernel the
// large-subset workload spends its time in).
//
// Method ("Dust：无需反向传播的Transformer零阶预训练", §1 减少干扰: the head is
// perturbed on cached logits and each draw evaluates a small subset of the
// vocabulary): draw i of token t perturbs logits j_k = (a k + b) mod V, k < S,
// plus the target; in the permuted column order q (logit a q mod V) the drawn
// set is the window [c, c+S) mod V, c = a^-1 b. LSE' = LSE +
// log1p(sum_drawn p_j expm1(sigma eps_j)), r = sigma eps_y - log1p(.), and
// r eps (scaled by the inverse inclusion probability) accumulates into g_t.
//
// B200 mapping: one cluster of CS CTAs (one per SM; CS = 1 or 2 where the
// slices fit in shared memory, else the size of 3 to 8 whose clusters cover
// the most SMs) per token at a time,
// persistent over tokens. CTA r of the cluster holds the probability row and
// the g accumulator for its slice [r seg, (r+1) seg) of q in shared memory
// (CS = 2 at V = 50304: 2 x 100.6 KB per CTA; CS = 8 reaches V ~ 223k), so
// the hot loop touches no global memory. A draw's S slots are NB blocks of
// 128 per warp (S <= 1024, NB <= 8). Warps take batches of 32 draws from
// a shared counter; in a batch each lane works out one draw's window start,
// whether its window holds the target and the noise of the appended target
// slot, and the warp then processes, one after the other, the draws whose
// window starts in its CTA's slice. With few draws (K <= 512, S <= 256) the
// draws of a token are set up together instead, the CTA's own collected in a
// shared list that is dealt out to the warps in turn (LIST). A window is no longer than a slice, so
// the part that runs past the slice (or wraps past V, which only a window
// starting in the last slice can do) lies in the next CTA's slice,
// (r + 1) mod CS, reached through DSMEM. The noise of a draw is generated
// once, already multiplied by sigma, kept in registers from the reward to the
// accumulation, and the first two Philox rounds are evaluated once per draw
// and once per slot block (they depend on the draw index or on the slot block
// only).
//
// Accumulation (INT = true): off-target coordinates accumulate r * sigma eps
// in 2^-15 fixed point (scaled by 1/sigma^2) with native int32 shared-memory
// atomics. |r| <= 11.54 sigma and |sigma eps| <= 5.77 sigma bound a term by
// 66.6 units-of-one, 2.2e6 < 2^22 fixed-point units, so the rounding to an
// integer is the exponent-bias construction fma(x, scale, 1.5 2^23) (the FMA
// pipe rounds to nearest, no conversion instruction). Sums wrap modulo 2^32,
// so only the final per-coordinate sum has to fit, which holds with a wide
// margin for K <= 65536 (a coordinate lies in about K S / V windows, and the
// scale shrinks as 16384/K above 16384 draws). The target coordinate, which
// collects all K draws, keeps an fp32 accumulator per warp. INT = false
// accumulates in fp32 (compare-and-swap atomics) for larger K.
//
// Token pipeline (rows of 16-byte multiples, V % 4 == 0): a CTA's slice of
// the next token's Z row is prefetched into L2 while the current token's
// draws run, and copied into shared memory by one bulk copy as soon as the
// draws are done, so that it lands while the g slice is written out (the
// write pass also clears the accumulator). Without it every token began with
// a chain of dependent global loads per thread, about a third of the launch
// at K = 1024. The wait for the copy is bounded: on expiry the kernel raises
// the timeout bit of the status word and runs on without waiting again.
#include <cooperative_groups.h>
#include <mutex>

#include "internal.cuh"
#include "noise.cuh"
#include "tc_ptx.cuh"

namespace cg = cooperative_groups;

namespace dust {
namespace {

// Threads per CTA. The fixed-point kernel with a series expm1 fits 64
// registers, so it runs 32 warps per SM (8 per scheduler), which hides the
// dependent-issue latency of the generator better than 16 warps at 116
// registers (4.5% less time at 32 than at 16 warps on the large-subset
// workload); the fp32-accumulator variant and the library expm1 (large sigma)
// keep 16 warps, where they need no spills.
// NB = 3 (the packed Box-Muller step, the tightest variant) also keeps 16
// warps: at 64 registers it spills whatever else the kernel holds. So do
// NB = 5 to 8 (S up to 1024), whose draws hold 20 to 32 noise values a lane;
// their ragged-S forms with the library expm1 or fp32 accumulators need more
// than 128 registers and run 12 warps (8 at NB = 7, 8 with the library expm1).
// The draw-list variants of NB = 3 and 4 (clusters of 3 to 8 CTAs) run 16
// warps too: the list's setup leaves them no register to spare at 64.
__host__ __device__ constexpr int sub2_threads(bool use_int, int deg, int nb, bool full,
                                               bool list) {
  return nb >= 5 ? (!full && (deg == 0 || !use_int) ? (nb >= 7 && deg == 0 ? 256 : 384) : 512)
                 : (use_int && deg != 0 && nb != 3 && !(list && nb >= 3) ? 1024 : 512);
}

// The Box-Muller step of NB-block draws in packed fp32x2 form, else scalar
// and paired up afterwards for the packed expm1 and accumulation. The packed
// operations run on the FMA-heavy pipe, which the Philox multiplies already
// load, so the scalar step (whose operations also use the FMA-lite pipe) is
// the faster one (0.3-0.7% on B200); at NB = 3 it needs more than the 64
// registers of a 1024-thread CTA, and those variants take the packed form, as
// do the 512-thread variants of NB = 5 to 8.
template <int NB>
constexpr bool packed_generator() { return NB == 3 || NB >= 5; }

constexpr int64_t kStaticSmem = 1024 + 8 * kSinCosTable;  // counters, angle table

struct Sub2Args {
  Key key;
  RoundKeys keys;
  uint32_t t_off, i_off, ctr3, stream_id;
  float sigma;
  int64_t T, V;
  int32_t K, S;
  uint32_t a, a_inv;
  uint64_t minv;  // floor((2^64 - 1) / V)
  uint32_t cs;    // CTAs per cluster
  uint32_t seg;   // q-slice length owned by one CTA (multiple of 4)
  float scale_other, scale_target;
  float fac;        // g = fac * sum r * (sigma eps)            (fp32 accumulators)
  float acc_scale;  // fixed-point units per unit of r * (sigma eps)
  float fac_int;    // g = fac_int * fixed-point sum
  uint32_t* status;  // kStatusTimeout when a row copy does not arrive
  const float* Z;    // clean logits, permuted columns (T x V)
  const float* lse;  // T
  const int32_t* y;
  float* rewards;
  float* g_out;
  void* gop;
  GopFormat gf;
  int64_t plane;
  // g = accumulator * w_other off the target; on it s_tgt * w_target (fixed
  // point) or its accumulator * w_target (fp32)
  float w_other, w_target;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// x y mod m for x, y < m < 2^31, with minv = floor((2^64 - 1) / m): the
// quotient estimate hi64(x y minv) is the true quotient or one less
// (Barrett), so one conditional subtraction ends it.
__device__ __forceinline__ uint32_t mulmod(uint32_t x, uint32_t y, uint32_t m, uint64_t minv) {
  const uint64_t p = (uint64_t)x * y;
  const uint64_t r = p - __umul64hi(p, minv) * m;
  return (uint32_t)(r >= m ? r - m : r);
}

template <bool INT>
__device__ __forceinline__ void accumulate(float* slot, float r, float x, float acc_scale) {
  if (INT)
    atomicAdd(reinterpret_cast<int*>(slot),
              __float_as_int(fmaf(r * acc_scale, x, 12582912.0f)) - 0x4B400000);
  else
    atomicAdd(slot, r * x);
}

// NB: 128-slot blocks per draw (S <= 128 NB); FULL: S == 128 NB; LIST: the
// per-token draw list (its 16-byte entries follow the slices in shared memory).
template <int NB, bool FULL, int DEG, bool INT, bool LIST>
__global__ __launch_bounds__(sub2_threads(INT, DEG, NB, FULL, LIST), 1) void k_subset2(const __grid_constant__ Sub2Args A) {
  constexpr int kThreads = sub2_threads(INT, DEG, NB, FULL, LIST);
  extern __shared__ __align__(16) float smem[];
  __shared__ int s_next;    // next draw batch of the current token
  __shared__ int s_cnt;     // LIST: entries of the current token's draw list
  __shared__ float s_tgt;   // INT: sum r * (sigma eps_y) of the target coordinate
  __shared__ float2 s_tab[kSinCosTable];
  __shared__ __align__(8) uint64_t s_row;  // completion of the row copy
  __shared__ float s_lse_n;                // LSE and target of the next token
  __shared__ int32_t s_y_n;
  __shared__ const float* s_row_n;         // its Z slice to copy (null: none)
  __shared__ uint32_t s_phase;             // phase of s_row the next row completes
  fill_sincos_table(s_tab, A.sigma);
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&s_row), 1);
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  __syncthreads();
  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t cs = A.cs;
  const uint32_t rank = cluster.block_rank();
  const int lane = threadIdx.x & 31;
  const uint32_t V = (uint32_t)A.V;
  const uint32_t seg = A.seg;
  const uint32_t lo = rank * seg;
  const uint32_t hi = min(V, lo + seg);
  const uint32_t n_own = hi - lo;
  const uint32_t peer = rank + 1 == cs ? 0u : rank + 1;  // holds the slice after this one
  const uint32_t lo_peer = peer * seg;
  float* sp = smem;        // p of q in [lo, hi)
  float* sg = smem + seg;  // g accumulator of q in [lo, hi) (fp32 or int32 fixed point)
  // the next CTA's p and g slices (DSMEM). NB = 2 and 3 read their
  // addresses from shared memory where a window crosses into them: held in
  // registers they push those variants past the 64 registers of a
  // 1024-thread CTA. NB = 1 and 4 keep them in registers (1.4 % faster on the
  // large-subset workload than reading them from shared memory), and so do the
  // 512-thread NB = 5 to 8.
  constexpr bool kPeerRegs = NB == 1 || NB >= 4;
  __shared__ float* s_peer[2];
  float* sp_peer = nullptr;
  float* sg_peer = nullptr;
  if constexpr (kPeerRegs) {
    sp_peer = cluster.map_shared_rank(sp, peer);
    sg_peer = cluster.map_shared_rank(sg, peer);
  } else {
    if (threadIdx.x == 0) {
      s_peer[0] = cluster.map_shared_rank(sp, peer);
      s_peer[1] = cluster.map_shared_rank(sg, peer);
    }
    __syncthreads();
  }
  auto peer_p = [&]() { return kPeerRegs ? sp_peer : *(float* volatile*)&s_peer[0]; };
  auto peer_g = [&]() { return kPeerRegs ? sg_peer : *(float* volatile*)&s_peer[1]; };
  const int S = A.S;
  const uint32_t nclusters = gridDim.x / cs;
  const uint32_t cid = blockIdx.x / cs;
  const int nbatch = (A.K + 31) >> 5;

  BlockConst bc[NB];
#pragma unroll
  for (int m = 0; m < NB; ++m) bc[m] = block_const(A.keys, slot_ctr0((uint32_t)m, (uint32_t)lane), A.ctr3);
  const bool vec = (V & 3u) == 0;  // rows start 16-byte aligned
  // the pipelined row copy (one bulk copy of n_own floats; 16-byte aligned
  // source and size when V % 4 == 0, the slices being multiples of 4)
  const bool bulk = vec;
  // thread 0: copy a slice of n_own floats at src into sp (every generic
  // access to sp of the previous token is ordered before the barrier that
  // precedes this)
  auto issue_row = [&](const float* src) {
    const uint32_t bar = ptx::smem_u32(&s_row);
    ptx::fence_proxy_async();
    ptx::mbar_expect_tx(bar, n_own * 4u);
    ptx::bulk_load(ptx::smem_u32(sp), src, n_own * 4u, bar);
  };

  if (bulk) {
    if (threadIdx.x == 0 && (int64_t)cid < A.T) issue_row(A.Z + (int64_t)cid * A.V + lo);
    for (uint32_t q = threadIdx.x * 4; q < n_own; q += kThreads * 4)
      *reinterpret_cast<float4*>(sg + q) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // the LSE and target of a token are loaded a token ahead (thread 0, into
  // shared memory, read after the barrier that ends the previous token)
  if (threadIdx.x == 0) s_cnt = 0;
  if (threadIdx.x == 0 && (int64_t)cid < A.T) {
    s_lse_n = A.lse[cid];
    s_y_n = A.y[cid];
    s_phase = 0;
  }
  __syncthreads();

  for (int64_t t = cid; t < A.T; t += nclusters) {
    const float lse_t = s_lse_n;
    int32_t yt = s_y_n;
    // ---- p = exp(z - LSE) for the owned slice (and clear g without bulk),
    // by the hardware exponential: its relative error, about 1e-6 at
    // z - LSE = -20 and less nearer 0, moves the reward sum by under 1e-7
    const float* zrow = A.Z + t * A.V;
    if (bulk) {
      // thread 0 waits for the row (the k-th token of this cluster for
      // phase k & 1), the block barrier passes its arrival on; once a wait
      // has expired (the status word says so) none waits again
      if (threadIdx.x == 0) {
        const uint32_t row_bar = ptx::smem_u32(&s_row);
        const uint32_t row_phase = s_phase;
        s_phase = row_phase ^ 1u;
        if (!(*(volatile uint32_t*)A.status & kStatusTimeout)) {
          bool ok = ptx::mbar_try_wait(row_bar, row_phase);
          if (!ok) {
            const uint64_t t0 = ptx::globaltimer_ns();
            for (uint32_t it = 1; !ok; ++it) {
              ok = ptx::mbar_try_wait(row_bar, row_phase);
              if (!ok && (it & 63u) == 0 && ptx::globaltimer_ns() - t0 > 2000000000ull) break;
            }
          }
          if (!ok) atomicOr(A.status, kStatusTimeout);
        }
      }
      __syncthreads();
      for (uint32_t q = threadIdx.x * 4; q < n_own; q += kThreads * 4) {
        const float4 z = *reinterpret_cast<const float4*>(sp + q);
        *reinterpret_cast<float4*>(sp + q) =
            make_float4(__expf(z.x - lse_t), __expf(z.y - lse_t), __expf(z.z - lse_t), __expf(z.w - lse_t));
      }
    } else for (uint32_t q = threadIdx.x * 4; q < n_own; q += kThreads * 4) {
      if (vec && q + 3 < n_own) {
        const float4 z = *reinterpret_cast<const float4*>(zrow + lo + q);
        *reinterpret_cast<float4*>(sp + q) =
            make_float4(__expf(z.x - lse_t), __expf(z.y - lse_t), __expf(z.z - lse_t), __expf(z.w - lse_t));
        *reinterpret_cast<float4*>(sg + q) = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        for (uint32_t u = q; u < n_own && u < q + 4; ++u) {
          sp[u] = __expf(zrow[lo + u] - lse_t);
          sg[u] = 0.0f;
        }
      }
    }
    if (threadIdx.x == 0) {
      s_next = 0;
      s_tgt = 0.0f;
    }
    if (yt < 0 || (int64_t)yt >= A.V) yt = 0;  // reported by the loss kernel
    const uint32_t qy = mulmod((uint32_t)yt, A.a_inv, V, A.minv);
    const uint32_t owner_y = qy / seg;  // the CTA whose slice holds the target
    float* gy = cluster.map_shared_rank(sg, owner_y) + (qy - owner_y * seg);
    const uint32_t t_abs = A.t_off + (uint32_t)t;
    // Setup of draw iq (one lane): its window start in permuted order, the
    // target's slot in the window, and whether the window starts in this
    // CTA's slice; for those, the noise of the appended target slot.
    auto setup = [&](int iq, uint32_t& c, uint32_t& kyq, float& x_extra) -> bool {
      const uint32_t i_abs = A.i_off + (uint32_t)iq;
      const uint32_t b = subset_offset(A.key, t_abs, i_abs, A.stream_id, V);
      c = mulmod(b, A.a_inv, V, A.minv);
      const bool mine = (c >= lo) && (c < hi);
      kyq = (qy >= c) ? qy - c : qy + V - c;
      x_extra = 0.0f;
      if (mine && kyq >= (uint32_t)S) {
        // the appended target slot S: counter block S >> 7, lane S & 31,
        // word (S >> 5) & 3 (its block constants formed here, once per
        // batch and lane, rather than held in registers)
        const BlockConst bs = block_const(A.keys, slot_ctr0((uint32_t)S >> 7, (uint32_t)S & 31u), A.ctr3);
        const uint32_t s_word = ((uint32_t)S >> 5) & 3u;
        const U4 w = philox_from2(bs, draw_const(A.keys, t_abs, i_abs), A.keys);
        const float2 nn = box_muller_tab(s_word < 2 ? w.x : w.z, s_word < 2 ? w.y : w.w, s_tab);
        x_extra = (s_word & 1u) ? nn.y : nn.x;
      }
      return mine;
    };
    if constexpr (LIST) {
      // every draw set up at once, the ones whose window starts in this
      // CTA's slice appended to the list (one atomic per warp)
      uint4* s_list = reinterpret_cast<uint4*>(smem + 2 * seg);
      for (int iq0 = (int)(threadIdx.x & ~31u); iq0 < A.K; iq0 += kThreads) {
        const int iq = iq0 + lane;
        uint32_t c = 0, kyq = 0;
        float xe = 0.0f;
        const bool mine = iq < A.K && setup(iq, c, kyq, xe);
        const uint32_t m = __ballot_sync(0xffffffffu, mine);
        int base = 0;
        if (lane == 0 && m) base = atomicAdd(&s_cnt, __popc(m));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (mine)
          s_list[base + __popc(m & ((1u << lane) - 1u))] =
              make_uint4((uint32_t)iq, c, kyq, __float_as_uint(xe));
      }
    }
    cluster.sync();
    // p of the target, from the owner's shared memory
    const float py = cluster.map_shared_rank(sp, owner_y)[qy - owner_y * seg];
    if (threadIdx.x == 0) {
      const int64_t tn = t + nclusters;
      const float* zn = nullptr;
      if (tn < A.T) {
        zn = A.Z + tn * A.V + lo;
        if (bulk) ptx::bulk_prefetch_l2(zn, n_own * 4u);
        s_lse_n = A.lse[tn];
        s_y_n = A.y[tn];
      }
      s_row_n = bulk ? zn : nullptr;
    }

    float tgt_acc = 0.0f;  // INT: this warp's sum r * (sigma eps_y), lane 0
    // Draw i with window start cw, target slot ky and appended-slot noise xe,
    // by the whole warp: reward, then accumulation into g.
    auto draw = [&](int i, uint32_t cw, uint32_t ky, float xe) {
      const DrawConst dc = draw_const(A.keys, t_abs, A.i_off + (uint32_t)i);
      const bool in_win = ky < (uint32_t)S;
      const bool local = (cw + (uint32_t)S) <= hi;  // whole window in this slice
      float n[NB][4];  // sigma * eps of the draw's slots
      float s = 0.0f;
      // packed fp32x2 generation and accumulation (at NB = 2 they need more
      // than the 64 registers of a 1024-thread CTA, so those variants keep
      // the scalar form)
      constexpr bool kPacked = NB != 2;
      if (local && kPacked) {
        // packed pairs: slots (lane, lane + 64) and (lane + 32, lane + 96)
        // of each block, words (0, 2) and (1, 3) of its counter
        const float* pw = sp + (cw - lo) + lane;
        float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int m = 0; m < NB; ++m) {
          const int k0 = m * 128 + lane;
          const bool u0 = FULL || k0 < S, u1 = FULL || k0 + 32 < S;
          const bool u2 = FULL || k0 + 64 < S, u3 = FULL || k0 + 96 < S;
          const float2 p02 = make_float2(u0 ? pw[m * 128] : 0.0f, u2 ? pw[m * 128 + 64] : 0.0f);
          const float2 p13 = make_float2(u1 ? pw[m * 128 + 32] : 0.0f, u3 ? pw[m * 128 + 96] : 0.0f);
          float2 e02, e13;
          if (packed_generator<NB>()) {
            gauss4_tab_x2(philox_from2(bc[m], dc, A.keys), s_tab, e02, e13);
          } else {
            const G4 g = gauss4_tab(philox_from2(bc[m], dc, A.keys), s_tab);
            e02 = make_float2(g.v[0], g.v[2]);
            e13 = make_float2(g.v[1], g.v[3]);
          }
          if (!FULL) {
            e02 = make_float2(u0 ? e02.x : 0.0f, u2 ? e02.y : 0.0f);
            e13 = make_float2(u1 ? e13.x : 0.0f, u3 ? e13.y : 0.0f);
          }
          n[m][0] = e02.x;
          n[m][1] = e13.x;
          n[m][2] = e02.y;
          n[m][3] = e13.y;
          s2 = __ffma2_rn(p02, expm1_small_x2<DEG>(e02), s2);
          s2 = __ffma2_rn(p13, expm1_small_x2<DEG>(e13), s2);
        }
        s = s2.x + s2.y;
      } else if (local) {
        const float* pw = sp + (cw - lo) + lane;
        float pv[NB][4];
#pragma unroll
        for (int m = 0; m < NB; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = m * 128 + lane + 32 * j;
            pv[m][j] = (FULL || k < S) ? pw[m * 128 + 32 * j] : 0.0f;
          }
#pragma unroll
        for (int m = 0; m < NB; ++m) {
          const G4 g = gauss4_tab(philox_from2(bc[m], dc, A.keys), s_tab);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = m * 128 + lane + 32 * j;
            const float x = (FULL || k < S) ? g.v[j] : 0.0f;
            n[m][j] = x;
            s = fmaf(pv[m][j], expm1_small<DEG>(x), s);
          }
        }
      } else {
#pragma unroll
        for (int m = 0; m < NB; ++m) {
          const G4 g = gauss4_tab(philox_from2(bc[m], dc, A.keys), s_tab);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = m * 128 + lane + 32 * j;
            float x = 0.0f;
            if (FULL || k < S) {
              uint32_t q = cw + (uint32_t)k;
              if (q >= V) q -= V;
              const float pq = (q >= lo && q < hi) ? sp[q - lo] : peer_p()[q - lo_peer];
              x = g.v[j];
              s = fmaf(pq, expm1_small<DEG>(x), s);
            }
            n[m][j] = x;
          }
        }
      }
      float xy;
      if (in_win) {
        const int my = (int)(ky >> 7), jy = (int)((ky >> 5) & 3u);
        const bool owner = lane == (int)(ky & 31u);
        float cand = 0.0f;
#pragma unroll
        for (int m = 0; m < NB; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (m == my && j == jy) {
              cand = n[m][j];
              // INT: the target coordinate is accumulated in fp32 below
              if (INT && owner) n[m][j] = 0.0f;
            }
        xy = __shfl_sync(0xffffffffu, cand, (int)(ky & 31u));
      } else {
        xy = xe;
        if (lane == 0) s = fmaf(py, expm1_small<DEG>(xy), s);
      }
      // a series expm1 bounds |s| by e^0.06 - 1: the fixed-point warp sum applies
      s = DEG != 0 ? warp_sum_fixed34(s) : warp_sum(s);
      const float r = xy - log1p_small(s);
      if (A.rewards && lane == 0) A.rewards[t * A.K + i] = r;
      if (local && INT && kPacked) {
        // fixed point as in accumulate<true>, two slots per packed FMA
        float* gw = sg + (cw - lo) + lane;
        const float ra = r * A.acc_scale;
        const float2 ra2 = make_float2(ra, ra), bias = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
        for (int m = 0; m < NB; ++m) {
          const int k0 = m * 128 + lane;
          const float2 a02 = __ffma2_rn(ra2, make_float2(n[m][0], n[m][2]), bias);
          const float2 a13 = __ffma2_rn(ra2, make_float2(n[m][1], n[m][3]), bias);
          int* g = reinterpret_cast<int*>(gw + m * 128);
          if (FULL || k0 < S) atomicAdd(g, __float_as_int(a02.x) - 0x4B400000);
          if (FULL || k0 + 32 < S) atomicAdd(g + 32, __float_as_int(a13.x) - 0x4B400000);
          if (FULL || k0 + 64 < S) atomicAdd(g + 64, __float_as_int(a02.y) - 0x4B400000);
          if (FULL || k0 + 96 < S) atomicAdd(g + 96, __float_as_int(a13.y) - 0x4B400000);
        }
      } else if (local) {
        float* gw = sg + (cw - lo) + lane;
#pragma unroll
        for (int m = 0; m < NB; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = m * 128 + lane + 32 * j;
            if (FULL || k < S) accumulate<INT>(gw + m * 128 + 32 * j, r, n[m][j], A.acc_scale);
          }
      } else {
#pragma unroll
        for (int m = 0; m < NB; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = m * 128 + lane + 32 * j;
            if (FULL || k < S) {
              uint32_t q = cw + (uint32_t)k;
              if (q >= V) q -= V;
              float* dst = (q >= lo && q < hi) ? sg + (q - lo) : peer_g() + (q - lo_peer);
              accumulate<INT>(dst, r, n[m][j], A.acc_scale);
            }
          }
      }
      if (INT) {
        if (lane == 0) tgt_acc = fmaf(r, xy, tgt_acc);
      } else if (!in_win && lane == 0) {
        atomicAdd(gy, r * xy);
      }
    };
    if constexpr (LIST) {
      // the list dealt out in turn: entry j to warp j mod (warps per CTA),
      // so no warp runs more than one draw beyond another
      const uint4* s_list = reinterpret_cast<const uint4*>(smem + 2 * seg);
      const int cnt = s_cnt;
      for (int j = (int)(threadIdx.x >> 5); j < cnt; j += kThreads / 32) {
        const uint4 e = s_list[j];
        draw((int)e.x, e.y, e.z, __uint_as_float(e.w));
      }
    } else {
      for (;;) {
        int bidx = 0;
        if (lane == 0) bidx = atomicAdd(&s_next, 1);
        bidx = __shfl_sync(0xffffffffu, bidx, 0);
        if (bidx >= nbatch) break;
        const int iq = bidx * 32 + lane;
        uint32_t c = 0, kyq = 0;
        float x_extra = 0.0f;
        const bool mine = iq < A.K && setup(iq, c, kyq, x_extra);
        uint32_t mask = __ballot_sync(0xffffffffu, mine);
        while (mask) {
          const int src = __ffs(mask) - 1;
          mask &= mask - 1;
          draw(bidx * 32 + src, __shfl_sync(0xffffffffu, c, src), __shfl_sync(0xffffffffu, kyq, src),
               __shfl_sync(0xffffffffu, x_extra, src));
        }
      }
    }
    if (INT && lane == 0) atomicAdd(cluster.map_shared_rank(&s_tgt, owner_y), tgt_acc);
    cluster.sync();
    if (LIST && threadIdx.x == 0) s_cnt = 0;  // every warp has read this token's count
    // no CTA of the cluster reads sp any more: the next row can come in
    if (threadIdx.x == 0 && s_row_n) issue_row(s_row_n);

    // ---- scale and write the owned slice of g, and clear it for the next
    // token: four entries per step for the fp16 operand of 16-byte rows
    // (one shared-memory read and clear, one 8-byte store), else one
    // (NB <= 2 only: NB = 3 and 4 have no registers to spare around their
    // draw loop, and at their sizes the pass is a smaller share of a token)
    bool vec_out = false;
    if constexpr (NB <= 2) vec_out = (V & 3u) == 0 && A.gf.kind == kGopF16;
    if constexpr (NB <= 2) if (vec_out) {
      // g = acc so, the target's from its own sum; the optional fp32 g in
      // vocabulary order first, while the accumulator is intact
      if (A.g_out) {
        for (uint32_t q = threadIdx.x; q < n_own; q += kThreads) {
          const uint32_t qg = lo + q;
          const float x = INT ? (float)reinterpret_cast<const int*>(sg)[q] : sg[q];
          A.g_out[t * A.V + mulmod(qg, A.a, V, A.minv)] =
              qg == qy ? (INT ? s_tgt : x) * A.w_target : x * A.w_other;
        }
        __syncthreads();  // every entry read before the loop below clears it
      }
      __half* orow = (__half*)A.gop + t * A.V + lo;
      for (uint32_t q = threadIdx.x * 4; q < n_own; q += kThreads * 4) {
        float4 a4 = *reinterpret_cast<const float4*>(sg + q);
        *reinterpret_cast<float4*>(sg + q) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (INT)
          a4 = make_float4((float)__float_as_int(a4.x), (float)__float_as_int(a4.y),
                           (float)__float_as_int(a4.z), (float)__float_as_int(a4.w));
        float v0 = a4.x * A.w_other, v1 = a4.y * A.w_other, v2 = a4.z * A.w_other,
              v3 = a4.w * A.w_other;
        if (qy - lo - q < 4u) {  // the target among these four
          const uint32_t j = qy - lo - q;
          const float vt =
              (INT ? s_tgt : (j == 0 ? a4.x : j == 1 ? a4.y : j == 2 ? a4.z : a4.w)) * A.w_target;
          v0 = j == 0 ? vt : v0;
          v1 = j == 1 ? vt : v1;
          v2 = j == 2 ? vt : v2;
          v3 = j == 3 ? vt : v3;
        }
        const __half2 h01 = __floats2half2_rn(v0 * A.gf.scale, v1 * A.gf.scale);
        const __half2 h23 = __floats2half2_rn(v2 * A.gf.scale, v3 * A.gf.scale);
        *reinterpret_cast<uint2*>(orow + q) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
      }
    }
    // one entry per step otherwise; the operand is fp16 (bf16 inputs) or
    // fp32, the launch takes no other, and each has a loop of its own
    auto entry = [&](uint32_t q) {
      const uint32_t qg = lo + q;
      float v;
      if (INT)
        v = (qg == qy) ? s_tgt * A.fac * A.scale_target
                       : (float)reinterpret_cast<const int*>(sg)[q] * A.fac_int * A.scale_other;
      else
        v = sg[q] * (qg == qy ? A.scale_target : A.scale_other) * A.fac;
      sg[q] = 0.0f;
      if (A.g_out) A.g_out[t * A.V + mulmod(qg, A.a, V, A.minv)] = v;
      return v;
    };
    if (!vec_out && A.gf.kind == kGopF16) {
      for (uint32_t q = threadIdx.x; q < n_own; q += kThreads)
        ((__half*)A.gop)[t * A.V + lo + q] = __float2half_rn(entry(q) * A.gf.scale);
    } else if (!vec_out) {
      for (uint32_t q = threadIdx.x; q < n_own; q += kThreads)
        ((float*)A.gop)[t * A.V + lo + q] = entry(q);
    }
    __syncthreads();
  }
  cluster.sync();
}

template <int NB, bool FULL, int DEG, bool INT, bool LIST>
cudaError_t launch_one(cudaStream_t st, const Sub2Args& A, size_t smem, int sm_count) {
  auto fn = k_subset2<NB, FULL, DEG, INT, LIST>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int cs = (int)A.cs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(sub2_threads(INT, DEG, NB, FULL, LIST));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = sm_count / cs;
  cfg.gridDim = dim3((unsigned)(max_clusters * cs));
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, (void*)fn, &cfg) == cudaSuccess && active > 0)
    max_clusters = active;
  cudaGetLastError();
  int64_t nc = A.T < max_clusters ? A.T : max_clusters;
  cfg.gridDim = dim3((unsigned)(nc * cs));
  e = cudaLaunchKernelEx(&cfg, fn, A);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int NB, bool FULL, bool INT, bool LIST>
cudaError_t launch_deg(cudaStream_t st, const Sub2Args& A, size_t smem, int sm, int deg) {
  if (deg == 3) return launch_one<NB, FULL, 3, INT, LIST>(st, A, smem, sm);
  if (deg == 4) return launch_one<NB, FULL, 4, INT, LIST>(st, A, smem, sm);
  return launch_one<NB, FULL, 0, INT, LIST>(st, A, smem, sm);
}

template <bool INT, bool LIST>
cudaError_t launch_nb(cudaStream_t st, const Sub2Args& A, size_t smem, int sm, int deg) {
  const int nb = (A.S + 127) / 128;
  const bool full = (A.S % 128) == 0;
  switch (nb) {
    case 1: return full ? launch_deg<1, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<1, false, INT, LIST>(st, A, smem, sm, deg);
    case 2: return full ? launch_deg<2, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<2, false, INT, LIST>(st, A, smem, sm, deg);
    case 3: return launch_deg<3, false, INT, LIST>(st, A, smem, sm, deg);
    case 4: return full ? launch_deg<4, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<4, false, INT, LIST>(st, A, smem, sm, deg);
    case 5: if constexpr (!LIST) return full ? launch_deg<5, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<5, false, INT, LIST>(st, A, smem, sm, deg);
            return cudaErrorNotSupported;
    case 6: if constexpr (!LIST) return full ? launch_deg<6, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<6, false, INT, LIST>(st, A, smem, sm, deg);
            return cudaErrorNotSupported;
    case 7: if constexpr (!LIST) return full ? launch_deg<7, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<7, false, INT, LIST>(st, A, smem, sm, deg);
            return cudaErrorNotSupported;
    case 8: if constexpr (!LIST) return full ? launch_deg<8, true, INT, LIST>(st, A, smem, sm, deg) : launch_deg<8, false, INT, LIST>(st, A, smem, sm, deg);
            return cudaErrorNotSupported;
    default: return cudaErrorNotSupported;
  }
}

// q-slice length of one CTA of a cs-CTA cluster (a multiple of 4, so rows
// start 16-byte aligned in shared memory).
int64_t slice_len(int64_t V, int cs) { return ((V + cs - 1) / cs + 3) / 4 * 4; }

// Never launched: the occupancy query below asks it how many clusters of a
// size fit at once with one CTA per SM, which the GPCs' SM counts decide.
__global__ void k_cluster_probe() {}

// SMs that clusters of cs CTAs of one CTA per SM cover at once (0 if unknown),
// cached per device.
int cluster_sms(int cs, int max_smem_optin) {
  static std::mutex mu;
  static int cache[16][9] = {};
  int dev = 0, sms = 0;
  if (cs < 1 || cs > 8 || cudaGetDevice(&dev) != cudaSuccess || dev >= 16 ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev][cs]) return cache[dev][cs] > 0 ? cache[dev][cs] : 0;
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)((sms / cs > 0 ? sms / cs : 1) * cs));
  cfg.blockDim = dim3(32);
  cfg.dynamicSmemBytes = (size_t)max_smem_optin;  // one CTA per SM
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaFuncSetAttribute(k_cluster_probe, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           max_smem_optin) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, (void*)k_cluster_probe, &cfg) != cudaSuccess)
    n = 0;
  cudaGetLastError();
  cache[dev][cs] = n > 0 ? n * cs : -1;
  return n > 0 ? n * cs : 0;
}

}  // namespace

// Cluster size the shared-memory kernel would use (0: not applicable). The
// slices (p and g, 4 bytes each) must fit in shared memory, and every slice
// be at least S long, so that a window reaches at most the next slice. One
// CTA, or two, where they fit; else, of 3 to 8 CTAs, the size whose clusters
// cover the most SMs at once (clusters of 8 fit 15 times on a 148-SM B200,
// 120 SMs, while smaller ones fill more of each GPC), the smaller on a tie.
int subset2_cluster_size(int64_t V, int32_t S, int max_smem_optin) {
  if (S < 1 || S > 1024 || V >= (1LL << 31)) return 0;
  auto fits = [&](int cs) {
    const int64_t seg = slice_len(V, cs);
    const int64_t last = V - (cs - 1) * seg;  // the last (shortest) slice
    if (2 * seg * 4 + kStaticSmem > max_smem_optin) return false;
    return cs == 1 || (S <= seg && S <= last);
  };
  if (fits(1)) return 1;
  if (fits(2)) return 2;
  int best = 0, best_sms = 0, fallback = 0;
  for (int cs = 3; cs <= 8; ++cs) {
    if (!fits(cs)) continue;
    if (!fallback && (cs == 4 || cs == 8)) fallback = cs;
    const int n = cluster_sms(cs, max_smem_optin);
    if (n > best_sms) {
      best = cs;
      best_sms = n;
    }
  }
  return best ? best : fallback;
}

cudaError_t launch_subset2(cudaStream_t st, const dust_params& p, int64_t a, int64_t a_inv,
                           const float* Z, const float* lse, const int32_t* y, float* rewards,
                           float* g_out, void* gop, GopFormat gf, int max_smem_optin,
                           int sm_count, uint32_t* status) {
  const int cs = subset2_cluster_size(p.V, p.S, max_smem_optin);
  if (!status || gf.kind == kGopBf16Planes) return cudaErrorInvalidValue;
  if (!cs) return cudaErrorNotSupported;
  Sub2Args A;
  A.key = key_of(p.seed);
  A.keys = round_keys(p.seed);
  A.t_off = (uint32_t)p.token_offset;
  A.i_off = (uint32_t)p.draw_offset;
  A.ctr3 = ctr3_of(kTagHead, p.stream_id);
  A.stream_id = p.stream_id;
  A.sigma = p.sigma;
  A.T = p.T;
  A.V = p.V;
  A.K = p.K;
  A.S = p.S;
  A.a = (uint32_t)a;
  A.a_inv = (uint32_t)a_inv;
  A.minv = ~0ull / (uint64_t)p.V;
  A.cs = (uint32_t)cs;
  A.seg = (uint32_t)slice_len(p.V, cs);
  A.scale_other = (float)((double)p.V / (double)p.S);
  A.scale_target = (p.flags & DUST_FLAG_LITERAL_TARGET_SCALE) ? A.scale_other : 1.0f;
  // the accumulators hold sum r (sigma eps): g = -(1/(K sigma)) sum r eps
  const double s2 = (double)p.sigma * (double)p.sigma;
  A.fac = p.sigma > 0.0f ? (float)(-1.0 / ((double)p.K * s2)) : 0.0f;
  // fixed point: 2^15 units per unit of r eps / sigma, fewer above 16384 draws
  const double units = 32768.0 * (p.K > 16384 ? 16384.0 / (double)p.K : 1.0);
  A.acc_scale = p.sigma > 0.0f ? (float)(units / s2) : 0.0f;
  A.fac_int = p.sigma > 0.0f ? (float)(-1.0 / ((double)p.K * units)) : 0.0f;
  const bool use_int = p.K <= 65536;
  A.w_other = use_int ? A.fac_int * A.scale_other : A.fac * A.scale_other;
  A.w_target = A.fac * A.scale_target;
  A.status = status;
  A.Z = Z;
  A.lse = lse;
  A.y = y;
  A.rewards = rewards;
  A.g_out = g_out;
  A.gop = gop;
  A.gf = gf;
  A.plane = p.T * p.V;
  // the per-token draw list (16 bytes a draw) for up to 512 draws and
  // S <= 256, when it fits beside the slices. At that K a warp has at most
  // about 8 draws of a token, and a batch of 32 leaves the slowest warp
  // several draws behind (on B200 at S = 256: K = 32 1.56 -> 1.09 ms,
  // K = 128 1.86 -> 1.58, K = 512 2.84 -> 2.73 for 8192 tokens). At K = 1024
  // the list's longer draw loop (6 % more instructions) costs more than the
  // balance gains (4.11 -> 4.30 ms), and larger S keeps batches: those
  // variants have no registers to spare.
  // Clusters of 3 to 8 CTAs (the larger vocabularies) split a token's draws
  // finer still: there the list serves S <= 512 up to 256 draws a CTA.
  const size_t slices = (size_t)2 * A.seg * 4, list_bytes = (size_t)p.K * 16;
  const bool list = use_int &&
                    ((p.K <= 512 && p.S <= 256) || (cs >= 3 && p.S <= 512 && p.K <= 256 * cs)) &&
                    slices + list_bytes + (size_t)kStaticSmem <= (size_t)max_smem_optin;
  const size_t smem = slices + (list ? list_bytes : 0);
  const int deg = expm1_degree(p.sigma);
  if (!use_int) return launch_nb<false, false>(st, A, smem, sm_count, deg);
  return list ? launch_nb<true, true>(st, A, smem, sm_count, deg)
              : launch_nb<true, false>(st, A, smem, sm_count, deg);
}

}  // namespace dust
