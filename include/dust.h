/*
 * dust.h — C ABI of the Dust per-token activation-space gradient estimator
 * (B200, sm_100a).
 *
 * What is computed. For a linear layer y_t = W x_t with cached inputs x_t and
 * cached clean outputs, K draws add independent per-token Gaussian noise
 * sigma*eps_t^(i) to y_t; the downstream per-token loss is recomputed from
 * cached intermediates; the reward is the loss reduction
 * r_t^(i) = L_t(clean) - L_t(perturbed); the output-error estimate is
 * g_t = -(1/(K sigma)) sum_i r_t^(i) eps_t^(i) and the weight gradient is
 * G_W = sum_t g_t x_t^T. Sources: "Dust：无需反向传播的Transformer零阶预训练"
 * §1 (激活空间扰动, 无需反向传播的信用分配, 减少干扰) and "Dust: предобучение
 * трансформеров без обратного распространения ошибки" ("Механика такая").
 *
 * Conventions shared by every entry point:
 *  - Tensor arguments are DEVICE pointers owned by the caller, row-major,
 *    contiguous, 16-byte aligned, unless an entry point says HOST.
 *  - Floating inputs are fp32 (dtype DUST_F32) or bf16 bit patterns stored as
 *    uint16 (DUST_BF16). Outputs are always fp32.
 *  - Every call is enqueued on the context's stream. By default the call ends
 *    by reading back a device status word (one 4-byte copy and a stream
 *    synchronisation), so device-detected errors (a target outside [0, V))
 *    are returned by the call itself; DUST_FLAG_ASYNC skips that read and
 *    leaves the status for dust_check().
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns DUST_ERR_ARG and launches nothing.
 *  - The context owns its scratch memory (grown on demand, freed by
 *    dust_destroy). A context is not thread-safe; use one per thread.
 *  - A context belongs to the device given to dust_create. Every call that
 *    touches the GPU first makes that device current (cudaSetDevice) and
 *    leaves it current on return; the stream must belong to that device.
 *  - Noise is Philox4x32-10 keyed by (seed, token, draw, slot) and is never
 *    stored: slot k of (token t, draw i) is output word ((k>>5)&3) of counter
 *    (((k>>7)<<5)|(k&31), t+token_offset, i+draw_offset, tag|(stream_id<<8)),
 *    key (seed lo, seed hi), turned into N(0,1) by Box-Muller on 24-bit
 *    uniforms (words 0,1 -> cos, sin; words 2,3 -> cos, sin). Tags: 0 = head
 *    logits, 1 = subset offset, 2 = MLP up-projection, 3 = MLP
 *    down-projection, 4 = attention output projection, 5 / 6 / 7 = query /
 *    key / value projection.
 */
#ifndef DUST_H
#define DUST_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dust_ctx dust_ctx;

typedef enum {
  DUST_OK = 0,
  DUST_ERR_ARG = 1,          /* invalid argument: nothing was launched */
  DUST_ERR_CUDA = 2,         /* a CUDA runtime or driver call failed */
  DUST_ERR_OOM = 3,          /* scratch allocation failed */
  DUST_ERR_BOUNDS = 4,       /* device-detected out-of-range index (a target) */
  DUST_ERR_TIMEOUT = 5,      /* a bounded device wait expired */
  DUST_ERR_UNSUPPORTED = 6   /* valid but not supported (shape, device) */
} dust_status;

typedef enum { DUST_F32 = 0, DUST_BF16 = 1 } dust_dtype;

enum {
  /* Scale the target coordinate of subset draws by V/S like the others (the
     literal reading; biased). Default: 1 for the target, V/S otherwise. */
  DUST_FLAG_LITERAL_TARGET_SCALE = 1u << 0,
  /* Do not read back the device status word at the end of the call. */
  DUST_FLAG_ASYNC = 1u << 1
};

/* Variants accepted by dust_validate. */
enum { DUST_VARIANT_HEAD = 0, DUST_VARIANT_MLP = 1, DUST_VARIANT_ATTN = 2 };

typedef struct dust_params {
  int64_t T;            /* tokens in this call (>= 1) */
  int64_t d;            /* layer input width (head: hidden; MLP: model width) */
  int64_t V;            /* vocabulary size (>= 1) */
  int64_t d_ff;         /* MLP hidden width (MLP variant only) */
  int32_t K;            /* draws per token (>= 1) */
  int32_t S;            /* head: <= 0 full vocabulary, else subset size (<= V) */
  float sigma;          /* noise scale (>= 0, finite); 0 gives zero estimates */
  int32_t dtype;        /* dust_dtype of the floating inputs */
  uint64_t seed;        /* Philox key */
  int64_t token_offset; /* absolute index of token 0 (noise counter word 1) */
  int64_t draw_offset;  /* absolute index of draw 0 (noise counter word 2) */
  int64_t subset_a;     /* subset stride a (coprime to V); 0: smallest integer
                           >= V (sqrt5-1)/2 coprime to V */
  uint32_t stream_id;   /* layer id, < 2^24 (noise counter word 3 bits 8..31) */
  uint32_t flags;       /* DUST_FLAG_* */
} dust_params;

/* Create a context on CUDA device `device`, enqueuing on `cuda_stream`
   (a cudaStream_t; NULL = the legacy default stream). Environment variables
   read here select alternative kernels of the context (all give the same
   results within the parity tolerances): DUST_DISABLE_TC=1 runs every GEMM
   on CUDA cores; DUST_TC_PAIR=0 gives each tensor-core GEMM tile one CTA
   instead of a CTA pair; DUST_SUBSET_KERNEL=1 uses the L2-fed subset-draw
   kernel instead of the shared-memory one; DUST_FULL_KERNEL=2 runs
   full-vocabulary draws as a reward pass and a g pass (the noise generated
   twice) instead of one pass; DUST_FULL_SPLIT=0 keeps a one-pass call on
   the context's stream, where by default the last ~8 % of its tokens go to
   the two passes on the SMs that the one-pass clusters leave empty, from
   two streams of the context's own (high and low priority) that fork from
   and join `cuda_stream` inside the call. A CUDA graph captured from such a
   call keeps the order but not the priorities unless it is instantiated
   with node priorities. */
dust_status dust_create(dust_ctx** out, int device, void* cuda_stream);
dust_status dust_set_stream(dust_ctx* ctx, void* cuda_stream);
/* Frees the context's scratch memory and streams; waits for its streams first. */
void dust_destroy(dust_ctx* ctx);
/* Last error message of the context (never NULL). */
const char* dust_last_error(const dust_ctx* ctx);
const char* dust_status_string(dust_status s);
/* Host-only check of a parameter block for `variant` (no GPU needed).
   `msg` (may be NULL) receives a reason of at most `msg_len` bytes. */
dust_status dust_validate(const dust_params* p, int variant, char* msg, int msg_len);
/* Subset stride the library uses for these parameters (the default when
   p->subset_a == 0); 0 if the parameters are invalid. Host-only. */
int64_t dust_subset_stride(const dust_params* p);
/* Reads and clears the device status word after DUST_FLAG_ASYNC calls. */
dust_status dust_check(dust_ctx* ctx);

/*
 * LM-head estimator on cached logits ("Dust：无需反向传播的Transformer零阶预训练"
 * §1 减少干扰: the head is perturbed on cached logits and each draw evaluates a
 * small subset of the vocabulary; "不用反向传播训练Transformer：Dust零阶优化获突破":
 * only the affected loss is recomputed).
 *   H        T x d   layer input (hidden states), dtype
 *   W        V x d   head weight, dtype
 *   targets  T       int32 token ids in [0, V)
 *   G_out    V x d   fp32 estimated weight gradient sum_t g_t h_t^T   (or NULL)
 *   loss_out T       fp32 clean per-token cross-entropy (natural log) (or NULL)
 *   rewards_out T x K fp32 r[t*K + i] = L_t - L'_t,i                  (or NULL)
 *   g_out    T x V   fp32 output-error estimate g_t, vocabulary order  (or NULL)
 * Full vocabulary (S <= 0): eps covers all V logits. Subset (S > 0): slot
 * k < S perturbs logit (a k + b) mod V with b = floor(w0 V / 2^32), w0 the
 * first word of counter (0, t, i, 1|(stream_id<<8)); the target is always
 * included (as slot S when not drawn); g is scaled per coordinate by its
 * inverse inclusion probability (V/S; 1 for the target).
 * With bf16 inputs G_out is contracted on tensor cores from g as one fp16
 * plane scaled by a power of two (the noise bounds |g| by 66.6 times its
 * inclusion scale, so every value is in range) and from H as fp16 with a
 * power-of-two scale taken from its largest magnitude (exact for bf16 values
 * in fp16's normal range): about 3e-4 relative error (Frobenius) from the
 * rounding of g. fp32 inputs keep fp32 throughout.
 * Errors: DUST_ERR_ARG (validation), DUST_ERR_BOUNDS (a target outside
 * [0, V): outputs are then unspecified), DUST_ERR_OOM, DUST_ERR_CUDA,
 * DUST_ERR_TIMEOUT (a bounded device wait expired: a GEMM pipeline stage or a
 * subset-draw row copy; outputs unspecified, the context stays usable).
 */
dust_status dust_head_grad(dust_ctx* ctx, const dust_params* p,
                           const void* H, const void* W, const int32_t* targets,
                           float* G_out, float* loss_out, float* rewards_out,
                           float* g_out);

/* Same as dust_head_grad with every tensor argument in HOST memory (pinned
   memory gives the fastest copies). The inputs are copied to the device, the
   estimator runs, and the requested outputs are copied back before return. */
dust_status dust_head_grad_host(dust_ctx* ctx, const dust_params* p,
                                const void* H, const void* W, const int32_t* targets,
                                float* G_out, float* loss_out, float* rewards_out,
                                float* g_out);

/*
 * Hidden-MLP up-projection estimator ("Dust：无需反向传播的Transformer零阶预训练"
 * §1: noise on each linear layer's output; 减少干扰: layer types perturbed in
 * separate passes with unperturbed intermediates cached). Noise goes on
 * u = x W_up^T (d_ff entries per token); each draw recomputes
 * GELU(u + sigma eps) - GELU(u), the down-projection and the head from the
 * cached x, u and clean logits (exact-erf GELU, residual h = x + a W_down^T,
 * no norm, no bias). Inputs are bf16; the clean activations a, h enter the
 * tensor-core GEMMs as bf16 hi/lo planes (about 2^-17 relative), against
 * weights duplicated along the contraction. The per-draw deltas are split the
 * same way; for sigma <= 0.05 the delta GEMMs contract their hi planes only,
 * and each reward gets the lo planes' first-order effect,
 * lo(dh) . u_t + lo(da) . (W_down^T u_t) with u_t = W_head[y_t] - W_head^T p_t
 * (p_t the clean softmax): two per-token vectors formed once per call by two
 * GEMMs. What that drops is of second order (rewards within about 3e-6 at
 * sigma = 0.05); above 0.05 both planes are contracted.
 *   X        T x d     input, dtype        W_up   d_ff x d   dtype
 *   W_down   d x d_ff  dtype               W_head V x d      dtype
 *   targets  T int32
 *   G_up_out d_ff x d  fp32 sum_t g_t x_t^T   (or NULL)
 *   loss_out T         fp32 clean CE           (or NULL)
 *   rewards_out T x K  fp32                    (or NULL)
 *   g_out    T x d_ff  fp32                    (or NULL)
 * p->S must be <= 0 (all d_ff channels are perturbed).
 */
dust_status dust_mlp_grad(dust_ctx* ctx, const dust_params* p,
                          const void* X, const void* W_up, const void* W_down,
                          const void* W_head, const int32_t* targets,
                          float* G_up_out, float* loss_out, float* rewards_out,
                          float* g_out);

/*
 * Hidden-MLP down-projection estimator (same pages and sections as
 * dust_mlp_grad, the next layer type of the block). Noise goes on
 * W_down's output (d entries per token), which is the block output h, so each
 * draw recomputes only the head: dz = sigma eps W_head^T (sigma eps as bf16
 * hi/lo planes, the GEMM on the hi plane with the lo plane's first-order
 * effect added as in dust_mlp_grad for sigma <= 0.05),
 * r = dz_y - log1p(sum p expm1(dz)),
 * g_t = -(1/(K sigma)) sum_i r_i eps_i, and the weight gradient is taken
 * against the layer's cached input a = GELU(u) (fp32, CUDA cores).
 *   arguments and layouts as dust_mlp_grad, except
 *   G_down_out d x d_ff fp32 sum_t g_t a_t^T   (or NULL)
 *   g_out      T x d    fp32                    (or NULL)
 * Its noise has its own counter tag (3), distinct from the up-projection's.
 * Same validation and errors as dust_mlp_grad.
 */
dust_status dust_mlp_down_grad(dust_ctx* ctx, const dust_params* p,
                               const void* X, const void* W_up, const void* W_down,
                               const void* W_head, const int32_t* targets,
                               float* G_down_out, float* loss_out, float* rewards_out,
                               float* g_out);

/*
 * Attention output-projection estimator (same pages and sections: the layer
 * types of a block perturbed in separate passes on cached intermediates).
 * The perturbed layer is y = W_o o, whose output is written into the residual
 * x that enters the MLP block (x = r + W_o o). Noise on y therefore moves x,
 * and each draw recomputes the MLP block and the head from the cached x, u and
 * clean logits:
 *   du = sigma eps W_up^T,  da = GELU(u + du) - GELU(u),
 *   dh = sigma eps + da W_down^T,  dz = dh W_head^T.
 * The reward and g_t (d entries) are as for dust_mlp_down_grad.
 *   X        T x d     the residual entering the block (bf16)
 *   O        T x d_o   the projection's cached input o_t (bf16), d_o a multiple of 8
 *   W_up, W_down, W_head, targets as dust_mlp_grad
 *   G_o_out  d x d_o   fp32 sum_t g_t o_t^T   (or NULL)
 *   loss_out, rewards_out as dust_mlp_grad;  g_out T x d fp32 (or NULL)
 * The noise has its own counter tag (4). Same validation and errors as
 * dust_mlp_grad, plus DUST_ERR_ARG for a NULL or misaligned O or a bad d_o.
 */
dust_status dust_attn_out_grad(dust_ctx* ctx, const dust_params* p,
                               const void* X, const void* O, int64_t d_o,
                               const void* W_up, const void* W_down, const void* W_head,
                               const int32_t* targets, float* G_o_out, float* loss_out,
                               float* rewards_out, float* g_out);

/*
 * Attention-internals estimator ("Dust：无需反向传播的Transformer零阶预训练",
 * §1 无需反向传播的信用分配 and 减少干扰: the attention internals are rewarded
 * from the change of the attention output, and a draw recomputes only the
 * attention output; "不用反向传播训练Transformer：Dust零阶优化获突破": that
 * change is judged together with an error signal).
 * Noise sigma eps (D = n_heads head_dim entries) goes on one token's output of
 * the query, key or value projection (shape->which). The attention is causal
 * multi-head attention over independent sequences of seq_len tokens with
 * scores q.k / sqrt(head_dim). A draw's reward is the first-order loss
 * decrease of the attention outputs it moves,
 *   r = -sum_t <o'_t - o_t, e_t>,
 * over t = s for query noise on token s and over t >= s of the same sequence
 * for key or value noise; e is the caller's error signal at the attention
 * output. Then g_s = -(1/(K sigma)) sum_i r_i eps_i (D entries) and
 * G = sum_s g_s x_s^T against the projection's input x.
 *   p        T (a multiple of seq_len), d (the width of x), K, sigma, seed,
 *            token_offset, draw_offset, stream_id, dtype (of X); V, d_ff,
 *            subset_a are not used; S must be <= 0
 *   shape    seq_len in [1, 4096], n_heads >= 1, head_dim 32, 64 or 128
 *   X        T x d   the projection's input (p->dtype)
 *   Q, Kc, Vc T x D  fp32 cached projections, head h in columns
 *                    [h head_dim, (h+1) head_dim)
 *   E        T x D   fp32 error signal at the attention output
 *   G_out    D x d   fp32 (or NULL)
 *   rewards_out T x K fp32 (or NULL);  g_out T x D fp32 (or NULL)
 * All pointers are device pointers, row-major; inputs 16-byte aligned,
 * outputs 4-byte. The noise's counter tag is 5, 6 or 7 (query, key, value).
 * Query and key noise with head_dim 64 or 128 runs its dot products on the
 * tensor cores in fp16 hi/lo parts (about fp32 accuracy); the environment
 * variable DUST_ATTN_TC=0 selects the CUDA-core form instead.
 * Errors: DUST_ERR_ARG for bad parameters, shape or pointers;
 * DUST_ERR_UNSUPPORTED when seq_len needs more shared memory than the device
 * has, or (reported at the end of the call) when a query or key value lies
 * beyond +-32768 on the tensor-core form; DUST_ERR_CUDA / DUST_ERR_OOM as
 * elsewhere.
 */
enum { DUST_ATTN_Q = 0, DUST_ATTN_K = 1, DUST_ATTN_V = 2 };
typedef struct dust_attn_shape {
  int32_t seq_len;   /* L: tokens per sequence */
  int32_t n_heads;   /* H */
  int32_t head_dim;  /* d_h: 32, 64 or 128 */
  int32_t which;     /* DUST_ATTN_Q, DUST_ATTN_K or DUST_ATTN_V */
} dust_attn_shape;
dust_status dust_attn_grad(dust_ctx* ctx, const dust_params* p, const dust_attn_shape* shape,
                           const void* X, const float* Q, const float* Kc, const float* Vc,
                           const float* E, float* G_out, float* rewards_out, float* g_out);

/* Per-stage device timing: when enabled, each call records CUDA events on
   the context's stream between its stages (clean GEMM, log-sum-exp, draws,
   g, G_W GEMM...). dust_stage_times waits for the last call's final event
   and fills names[i] / ms[i] for i < cap; it returns the number of stages. */
dust_status dust_set_stage_timing(dust_ctx* ctx, int enable);
int dust_stage_times(dust_ctx* ctx, const char** names, float* ms, int cap);
/* Number of kernels the context has launched since it was created. */
int64_t dust_kernel_launches(const dust_ctx* ctx);

/*
 * The LM-head estimator without any allocation, for callers that cannot call
 * cudaMalloc: code whose device memory is entirely owned by another allocator
 * (a framework's caching allocator or a pre-reserved pool, where a fresh
 * cudaMalloc fails or fragments the pool), and latency-critical code that
 * cannot afford the device-wide synchronisation cudaMalloc and cudaFree can
 * cause. The Dust pages have no counterpart to this entry point; it computes
 * exactly what dust_head_grad computes (same arguments and outputs, all device
 * pointers owned by the caller, on `cuda_stream` of the current device).
 *   - No context and no allocation: all scratch (logits, log-sum-exp, partial
 *     sums, rewards, the g operand, the status word) lives in one fixed 16 MiB
 *     device array that every GPU loading this library holds until the
 *     process exits. Problems needing more scratch than that (roughly
 *     T * V <= 2M fp32 elements) return DUST_ERR_UNSUPPORTED with the needed
 *     size in `msg`; CUDA-core GEMMs only.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. The address is kept with the CUDA context
 *     current at that call: after the device's primary context is destroyed
 *     and created anew (cudaDeviceReset), the next call looks it up again,
 *     so make that call outside a capture too.
 *   - Every call shares the array, which keeps the previous call's contents
 *     (each call clears what must start at zero). Calls that overlap on the
 *     GPU, on any stream or thread, race on it: serialise them.
 *   - The call synchronises `cuda_stream` to read the device status word
 *     (DUST_FLAG_ASYNC in p->flags is ignored).
 * Errors as dust_head_grad, with the reason in `msg` (may be NULL): invalid
 * parameters, NULL inputs, H or W not 16-byte aligned or another pointer not
 * 4-byte aligned return DUST_ERR_ARG before any CUDA call.
 */
dust_status dust_head_grad_noalloc(const dust_params* p, void* cuda_stream,
                                   const void* H, const void* W, const int32_t* targets,
                                   float* G_out, float* loss_out, float* rewards_out,
                                   float* g_out, char* msg, int msg_len);

/* One step of SGD with momentum on n weights (the Dust pages train with SGD
   and momentum, "Dust：无需反向传播的Transformer零阶预训练" §2 实证发现, and
   leave its form open; this is the heavy-ball step without dampening,
   Nesterov term or weight decay):
     v <- mu v + G,   W <- W - lr v            (fp32, elementwise)
   G: the estimator's weight gradient (device, fp32, read only, e.g. G_out of
   dust_head_grad); v: momentum buffer (device, fp32, in/out; start it at
   zero); W: fp32 master weights (device, in/out); W_bf16: NULL, or a device
   bf16 array that receives W rounded to nearest even (the copy the next
   estimator call reads). G, v and W must not overlap one another; all three
   16-byte aligned, W_bf16 8-byte aligned (DUST_ERR_ARG otherwise, before any
   launch). Asynchronous on the context's stream; n = 0 launches nothing. */
dust_status dust_sgd_momentum(dust_ctx* ctx, int64_t n, float lr, float mu, const float* G,
                              float* v, float* W, void* W_bf16);

/* Debug: C (M x N, fp32, row-major) = A B^T for bf16 row-major A (M x K) and
   B (N x K), through the library's GEMMs: path 0 = automatic, 1 = CUDA cores,
   2 = tcgen05 tensor cores with one CTA per 128 x 256 tile, 3 = tcgen05 with
   CTA pairs (cta_group::2) per 256 x 256 tile (2 and 3 return
   DUST_ERR_UNSUPPORTED when the shape does not fit: K a multiple of 8 and
   N >= 16 are needed), 4 = path 2 with an injected failure: the pipeline's
   bounded waits give up at once, the kernel drains its copies and MMAs, frees
   its TMEM and returns, and the call reports DUST_ERR_TIMEOUT with C
   undefined (the context stays usable). Synchronous. */
dust_status dust_debug_gemm_bf16(dust_ctx* ctx, int64_t M, int64_t N, int64_t K, const void* A,
                                 const void* B, float* C, int path);
/* Debug: the same product with both operands stored MN-major: At (K x M,
   bf16, row-major) and Bt (K x N), C (M x N, fp32) = At^T Bt. The tensor-core
   paths read the K x M and K x N rows as stored (M and N multiples of 8 are
   needed for 16-byte rows; else paths 2 and 3 return DUST_ERR_UNSUPPORTED
   and path 0 runs on CUDA cores). Paths and errors as dust_debug_gemm_bf16.
   This is the layout of the weight-gradient contraction sum_t g_t x_t^T. */
dust_status dust_debug_gemm_bf16_mn(dust_ctx* ctx, int64_t M, int64_t N, int64_t K,
                                    const void* At, const void* Bt, float* C, int path);

/* Debug: raw Philox4x32-10 words. ctr4 (n x 4 uint32, device) -> out (n x 4). */
dust_status dust_debug_philox(dust_ctx* ctx, uint64_t seed, const uint32_t* ctr4,
                              int64_t n, uint32_t* out);
/* Debug: eps for tokens [0, nt), draws [0, ni), slots [0, nslots) of tag `tag`
   under p's seed, offsets and stream_id -> out[(t*ni + i)*nslots + k] fp32. */
dust_status dust_debug_gauss(dust_ctx* ctx, const dust_params* p, int32_t tag,
                             int64_t nt, int64_t ni, int64_t nslots, float* out);
/* Debug: the same eps through the table-driven angle step the LM-head draw
   kernels use (a 1024-entry table of roots of unity plus angle addition), in
   the packed fp32x2 form those kernels run (the two Box-Muller pairs of a
   Philox counter side by side); it agrees with dust_debug_gauss to a few
   1e-7. */
dust_status dust_debug_gauss_tab(dust_ctx* ctx, const dust_params* p, int32_t tag,
                                 int64_t nt, int64_t ni, int64_t nslots, float* out);
/* Debug: the table-driven step in scalar form, one Box-Muller pair at a
   time; equal to dust_debug_gauss_tab bit for bit (same operations, same
   rounding). */
dust_status dust_debug_gauss_tab_scalar(dust_ctx* ctx, const dust_params* p, int32_t tag,
                                        int64_t nt, int64_t ni, int64_t nslots, float* out);

/* Debug: the Box-Muller radius for every 24-bit input (the pages fix only
   Gaussian noise; this transform is the library's). out (2^24 fp32, device)
   receives, at index j, for u1 = (j + 1) 2^-24:
     method 0: sigma sqrt(-2 ln u1) as the polynomial angle step forms it
               (sigma sqrt(2 ln 2) times rho);
     method 1: rho = sqrt(-log2 u1), the factor the table angle step
               multiplies into its table (sigma is not used).
   sigma must be finite and >= 0. Synchronous. */
dust_status dust_debug_bm_radius(dust_ctx* ctx, int32_t method, float sigma, float* out);
/* Debug: the Box-Muller angle step for every 24-bit input. out (2 x 2^24
   fp32, device) receives at [2m, 2m+1], for the angle 2 pi m 2^-24:
     method 0: (cos, sin), the polynomial step (MLP noise);
     method 1: sqrt(2 ln 2) (cos, sin), the table step (LM-head noise) with
               sigma = 1, whose table carries the radius factor that rho
               leaves out.
   Synchronous. */
dust_status dust_debug_bm_angle(dust_ctx* ctx, int32_t method, float* out);

#ifdef __cplusplus
}
#endif

#endif /* DUST_H */
