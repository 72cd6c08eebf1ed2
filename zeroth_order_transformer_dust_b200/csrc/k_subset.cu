// Vocabulary-subset LM-head draws ("Dust：无需反向传播的Transformer零阶预训练",
// §1 减少干扰: "each draw evaluates only a small part of the vocabulary").
//
// Draw i of token t perturbs the S logits j_k = (a k + b) mod V (k < S) plus
// the target (slot S when it is not drawn). With the probability row stored
// in permuted order -- column q holds vocabulary index (a q) mod V -- the
// drawn set is the contiguous window q in [c, c + S) mod V with
// c = a^-1 b mod V, and slot k sits at q = c + k. The perturbed
// log-sum-exp is updated in place,
//   LSE' = LSE + log1p(sum_{j drawn} p_j expm1(sigma eps_j)),
// the reward is r = sigma eps_y - log1p(.), and r * eps is accumulated into
// the token's g row, which lives in shared memory for the whole token. The
// noise of a draw is generated once and kept in registers between the reward
// and the accumulation.
#include "internal.cuh"
#include "noise.cuh"

namespace dust {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

struct SubsetArgs {
  Key key;
  uint32_t t_off, i_off, ctr3, stream_id;
  float sigma;
  int64_t V;
  int32_t K, S;
  int64_t a, a_inv;
  float scale_other, scale_target, fac;
  const float* P;
  const int32_t* y;
  float* rewards;
  float* g_out;
  void* gop;
  float* gacc;  // global accumulator rows (only when the row does not fit in smem)
  GopFormat gf;
  int64_t plane;  // distance between the hi and lo planes of the bf16 operand
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t mulmod(uint64_t x, uint64_t y, uint64_t m) {
  return (uint32_t)((x * y) % m);
}

// NB: number of 128-slot blocks whose noise stays in registers; blocks
// beyond NB are regenerated for the accumulation.
template <int NB, int DEG, bool GSMEM>
__global__ __launch_bounds__(kThreads, 1) void k_subset(SubsetArgs A) {
  extern __shared__ float gs_dyn[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x;
  const int64_t V = A.V;
  const uint32_t Vu = (uint32_t)V;
  float* G = GSMEM ? gs_dyn : A.gacc + t * V;
  for (int64_t q = threadIdx.x; q < V; q += kThreads) G[q] = 0.0f;
  __syncthreads();

  int32_t yt = A.y[t];
  if (yt < 0 || (int64_t)yt >= V) yt = 0;  // reported by the loss kernel
  const uint32_t qy = mulmod((uint32_t)yt, (uint64_t)A.a_inv, V);
  const float* Pt = A.P + t * V;
  const float py = Pt[qy];
  const uint32_t t_abs = A.t_off + (uint32_t)t;
  const int S = A.S;
  const int nblk = (S + 127) >> 7;

  for (int i = warp; i < A.K; i += kWarps) {
    const uint32_t i_abs = A.i_off + (uint32_t)i;
    const uint32_t b = subset_offset(A.key, t_abs, i_abs, A.stream_id, Vu);
    const uint32_t c = mulmod(b, (uint64_t)A.a_inv, V);
    const uint32_t ky = (qy >= c) ? qy - c : qy + Vu - c;
    const bool in_win = ky < (uint32_t)S;
    float n[NB][4];
    float s = 0.0f;
#pragma unroll
    for (int m = 0; m < NB; ++m) {
      if (m < nblk) {
        U4 cc{slot_ctr0((uint32_t)m, (uint32_t)lane), t_abs, i_abs, A.ctr3};
        const G4 g = gauss4(philox10(cc, A.key.k0, A.key.k1));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int k = m * 128 + lane + 32 * j;
          float v = 0.0f;
          if (k < S) {
            uint32_t pos = c + (uint32_t)k;
            if (pos >= Vu) pos -= Vu;
            v = g.v[j];
            s = fmaf(Pt[pos], expm1_small<DEG>(A.sigma * v), s);
          }
          n[m][j] = v;
        }
      }
    }
    for (int m = NB; m < nblk; ++m) {
      U4 cc{slot_ctr0((uint32_t)m, (uint32_t)lane), t_abs, i_abs, A.ctr3};
      const G4 g = gauss4(philox10(cc, A.key.k0, A.key.k1));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = m * 128 + lane + 32 * j;
        if (k < S) {
          uint32_t pos = c + (uint32_t)k;
          if (pos >= Vu) pos -= Vu;
          s = fmaf(Pt[pos], expm1_small<DEG>(A.sigma * g.v[j]), s);
        }
      }
    }
    float ey;
    if (in_win) {
      // eps of the target slot ky lives in lane ky & 31, block ky >> 7, word (ky >> 5) & 3
      const int my = (int)(ky >> 7), jy = (int)((ky >> 5) & 3u);
      float cand = 0.0f;
      if (my < NB) {
#pragma unroll
        for (int m = 0; m < NB; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (m == my && j == jy) cand = n[m][j];
      } else {
        cand = gauss_slot(A.key, t_abs, i_abs, A.ctr3, ky);
      }
      ey = __shfl_sync(0xffffffffu, cand, (int)(ky & 31u));
    } else {
      ey = gauss_slot(A.key, t_abs, i_abs, A.ctr3, (uint32_t)S);
      if (lane == 0) s = fmaf(py, expm1_small<DEG>(A.sigma * ey), s);
    }
    s = warp_sum(s);
    const float r = A.sigma * ey - log1pf(s);
    if (A.rewards && lane == 0) A.rewards[t * A.K + i] = r;
#pragma unroll
    for (int m = 0; m < NB; ++m) {
      if (m < nblk) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int k = m * 128 + lane + 32 * j;
          if (k < S) {
            uint32_t pos = c + (uint32_t)k;
            if (pos >= Vu) pos -= Vu;
            atomicAdd(&G[pos], r * n[m][j]);
          }
        }
      }
    }
    for (int m = NB; m < nblk; ++m) {
      U4 cc{slot_ctr0((uint32_t)m, (uint32_t)lane), t_abs, i_abs, A.ctr3};
      const G4 g = gauss4(philox10(cc, A.key.k0, A.key.k1));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = m * 128 + lane + 32 * j;
        if (k < S) {
          uint32_t pos = c + (uint32_t)k;
          if (pos >= Vu) pos -= Vu;
          atomicAdd(&G[pos], r * g.v[j]);
        }
      }
    }
    if (!in_win && lane == 0) atomicAdd(&G[qy], r * ey);
  }
  __syncthreads();

  for (int64_t q = threadIdx.x; q < V; q += kThreads) {
    const float v = G[q] * ((uint32_t)q == qy ? A.scale_target : A.scale_other) * A.fac;
    store_gop(A.gop, A.gf, A.plane, t * V + q, v);
    if (A.g_out) A.g_out[t * V + mulmod((uint32_t)q, (uint64_t)A.a, V)] = v;
  }
}

template <int NB, bool GSMEM>
cudaError_t launch_nb(cudaStream_t st, const SubsetArgs& A, int64_t T, size_t smem, int deg) {
  void (*fn)(SubsetArgs);
  if (deg == 3) fn = k_subset<NB, 3, GSMEM>;
  else if (deg == 4) fn = k_subset<NB, 4, GSMEM>;
  else fn = k_subset<NB, 0, GSMEM>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  fn<<<(unsigned)T, kThreads, smem, st>>>(A);
  return cudaGetLastError();
}

template <bool GSMEM>
cudaError_t launch_g(cudaStream_t st, const SubsetArgs& A, int64_t T, size_t smem, int deg) {
  const int nblk = (A.S + 127) / 128;
  if (nblk <= 1) return launch_nb<1, GSMEM>(st, A, T, smem, deg);
  if (nblk <= 2) return launch_nb<2, GSMEM>(st, A, T, smem, deg);
  if (nblk <= 4) return launch_nb<4, GSMEM>(st, A, T, smem, deg);
  if (nblk <= 8) return launch_nb<8, GSMEM>(st, A, T, smem, deg);
  return launch_nb<16, GSMEM>(st, A, T, smem, deg);
}

}  // namespace

size_t subset_gacc_bytes(int64_t T, int64_t V, int max_smem_optin) {
  return (size_t)V * 4 <= (size_t)max_smem_optin ? 0 : (size_t)T * V * 4;
}

cudaError_t launch_subset_impl(cudaStream_t st, const dust_params& p, int64_t a, int64_t a_inv,
                               const float* P, const int32_t* y, float* rewards, float* g_out,
                               void* gop, GopFormat gf, float* gacc, int max_smem_optin) {
  SubsetArgs A;
  A.key = key_of(p.seed);
  A.t_off = (uint32_t)p.token_offset;
  A.i_off = (uint32_t)p.draw_offset;
  A.ctr3 = ctr3_of(kTagHead, p.stream_id);
  A.stream_id = p.stream_id;
  A.sigma = p.sigma;
  A.V = p.V;
  A.K = p.K;
  A.S = p.S;
  A.a = a;
  A.a_inv = a_inv;
  A.scale_other = (float)((double)p.V / (double)p.S);
  A.scale_target = (p.flags & DUST_FLAG_LITERAL_TARGET_SCALE) ? A.scale_other : 1.0f;
  A.fac = p.sigma > 0.0f ? -1.0f / ((float)p.K * p.sigma) : 0.0f;
  A.P = P;
  A.y = y;
  A.rewards = rewards;
  A.g_out = g_out;
  A.gop = gop;
  A.gacc = gacc;
  A.gf = gf;
  A.plane = p.T * p.V;
  const int deg = expm1_degree(p.sigma);
  const size_t smem = (size_t)p.V * 4;
  if (smem <= (size_t)max_smem_optin) return launch_g<true>(st, A, p.T, smem, deg);
  if (!gacc) return cudaErrorInvalidValue;
  return launch_g<false>(st, A, p.T, 0, deg);
}

}  // namespace dust
