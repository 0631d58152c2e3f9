/*
 * dg.h -- C ABI of the B200 denoising-step library for block-autoregressive
 * multinomial text diffusion with a top-k MoE (DiffusionGemma-style).
 *
 * Sources of the operations, cited by tag:
 *   [P1] DiffusionGemma technical-report summary (animattoys.com):
 *        section 一 (multinomial diffusion: noise replaces a token by a uniform
 *        vocabulary token; a 256-token random canvas; ~12 rounds on average),
 *        section 二 (Gemma-4 MoE, 128 experts / top-8; causal prompt encoding into
 *        the KV cache and bidirectional canvas attention; self-conditioning on the
 *        previous round's predictions with ~7.8M extra parameters),
 *        section 四 (the sampler: confidence, entropy, re-randomising the
 *        uncertain positions, temperature, adaptive stop on mean entropy, a
 *        48-round budget), section 五 (per-step cost: MoE, softmax over the
 *        262k vocabulary and the self-conditioning matmul, canvas attention).
 *   [P2] DiffusionGemma overview (youleyou.com), 架构基础 (causal encoder into
 *        the KV cache, bidirectional denoiser over the canvas, finished blocks
 *        handed to the KV cache) and 离散文本扩散的运作机制 (canvas init,
 *        iterative refinement, re-noising of low-confidence positions).
 *   [P3] "Google 開源 DiffusionGemma" (akiraxclaw.com): a finished canvas is
 *        encoded into the KV cache before the next one starts.
 *   [Philox] Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless the comment says host.  The caller
 *     owns every pointer it passes; the library never frees them.  Weights are
 *     BORROWED: they must stay valid and unchanged until dg_destroy.
 *   - Matrices are row-major [out, in] (the layout of a linear layer's weight).
 *   - Work is ordered on the handle's stream.  Entry points that return results
 *     on the host (steps_used, lengths) synchronise that stream.
 *   - Return value: DG_OK or an error code; dg_last_error() gives the message.
 *     All shape, alignment and capacity checks run on the host before any
 *     launch; a failed check launches nothing and leaves state unchanged.
 *     A device-side timeout in a kernel wait is reported as DG_ETIMEOUT by the
 *     next call that synchronises.  No entry point traps the device.
 *   - dtype DG_BF16: weights, activations between GEMMs and the KV cache are
 *     bf16, accumulation and the residual stream fp32.  dtype DG_FP32: all fp32.
 *     Norm weights and the router bias are fp32 in both.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  DG_OK = 0,
  DG_EINVAL = 1,     /* bad argument, shape, alignment or null pointer */
  DG_ENOMEM = 2,     /* device or pinned-host allocation failed */
  DG_ECUDA = 3,      /* a CUDA runtime/driver call failed */
  DG_ECAPACITY = 4,  /* KV cache or workspace capacity exceeded */
  DG_ESTATE = 5,     /* call not valid in the handle's state */
  DG_ETIMEOUT = 6    /* a bounded device-side wait gave up */
};

enum { DG_FP32 = 0, DG_BF16 = 1 };

typedef struct dg_handle dg_handle;

/* Model shape and capacities ([P1 二]). */
typedef struct dg_config {
  int n_layers;      /* transformer layers (0: sampler-only handle) */
  int d_model;       /* d */
  int n_heads;       /* Hq query heads */
  int n_kv_heads;    /* Hkv KV heads; Hq % Hkv == 0 (GQA) */
  int head_dim;      /* hd, even */
  int n_experts;     /* E <= 256 */
  int top_k;         /* k <= min(E, 16) */
  int d_ff;          /* F, expert FFN width */
  int vocab;         /* V */
  int canvas;        /* N, canvas length (256 in [P1 一]) */
  int max_batch;     /* request slots, 1..64 */
  int max_ctx;       /* KV capacity per request in positions, multiple of 64 */
  int max_tokens;    /* rows per forward pass (>= max_batch*canvas; 0 = that) */
  int dtype;         /* DG_BF16 or DG_FP32 */
  double rope_base;  /* RoPE base (10000) */
  double rms_eps;    /* RMSNorm epsilon */
  int expert_format; /* DG_EXPERT_DTYPE (0: experts in the handle's dtype) or DG_EXPERT_NVFP4 (bf16 handles) */
} dg_config;

/* Storage of the expert weights ([P2] 推荐的部署与优化方案 and [P4] MoE 26B参数架构分析:
 * the model ships NVFP4 weights for Blackwell).
 * DG_EXPERT_NVFP4: each expert matrix [out, in] (in a multiple of 64) is
 *   - codes: [out, in/2] bytes of FP4 E2M1 codes, element 2j in the low nibble
 *     of byte j (OCP MX E2M1: 1 sign, 2 exponent, 1 mantissa bit);
 *   - block scales: one E4M3 code per 16 consecutive elements of a row, stored
 *     tiled as [in/64][out_pad][4] bytes, out_pad = out rounded up to 128
 *     (entry [k/64][row][(k%64)/16]; padding rows are 0);
 *   - g: one fp32 scale per matrix;
 *   value = E2M1(code) * E4M3(scale) * g.  dg_quantize_nvfp4 produces it.
 * Activations stay bf16: the kernels expand the codes to bf16 (exact: at most
 * 6 significant bits) ahead of the bf16 tensor-core product and apply g to
 * the fp32 accumulator. */
enum { DG_EXPERT_DTYPE = 0, DG_EXPERT_NVFP4 = 1 };

/* One layer's weights (all borrowed device pointers). */
typedef struct dg_layer_weights {
  const float* attn_norm;  /* [d] fp32 */
  const void* wq;          /* [Hq*hd, d] */
  const void* wk;          /* [Hkv*hd, d] */
  const void* wv;          /* [Hkv*hd, d] */
  const void* wo;          /* [d, Hq*hd] */
  const float* ffn_norm;   /* [d] fp32 */
  const void* router_w;    /* [E, d] */
  const float* router_b;   /* [E] fp32, or NULL for no bias */
  const void* w_gate;      /* [E, F, d] */
  const void* w_up;        /* [E, F, d] */
  const void* w_down;      /* [E, d, F] */
  /* DG_EXPERT_NVFP4 only (w_gate / w_up / w_down then hold the codes [E, out, in/2]): */
  const uint8_t* w_gate_sf;  /* block scales [E][d/64][F_pad][4] */
  const uint8_t* w_up_sf;    /* [E][d/64][F_pad][4] */
  const uint8_t* w_down_sf;  /* [E][F/64][d_pad][4] */
  const float* w_gate_g;     /* [E] per-matrix fp32 scales */
  const float* w_up_g;       /* [E] */
  const float* w_down_g;     /* [E] */
} dg_layer_weights;

typedef struct dg_weights {
  const void* embed;                /* [V, d]; also the tied LM head */
  const void* w_sc;                 /* [d, d] self-conditioning projection */
  const float* final_norm;          /* [d] fp32 */
  const dg_layer_weights* layers;   /* HOST array of n_layers entries */
} dg_weights;

/* Sampler settings for one step ([P1 四]). */
typedef struct dg_sampler_params {
  float temperature;     /* T > 0; 0 = argmax (ties to the lower index) */
  float logit_scale;     /* s: statistics use z = s * logit / T */
  float stop_threshold;  /* stop when mean entropy (nats) < this; < 0 disables */
  int keep_k;            /* positions kept this step (0..N) */
  uint64_t seed;         /* Philox key */
  uint32_t block;        /* Philox counter word 2 (block index) */
  int keep_mode;         /* DG_KEEP_TOPK (0, the default when zeroed) or DG_KEEP_ENTROPY_BUDGET */
  float entropy_budget;  /* nats, >= 0; read only by DG_KEEP_ENTROPY_BUDGET */
  int stop_mode;         /* DG_STOP_MEAN_ENTROPY (0, the default) or DG_STOP_TWO_ROUNDS */
  const int32_t* prev_argmax;      /* DG_STOP_TWO_ROUNDS: device [B, N], the previous round's argmax
                                      output, or NULL at the first round */
  const float* prev_mean_entropy;  /* DG_STOP_TWO_ROUNDS: device [B], the previous round's mean
                                      entropy, or NULL at the first round */
} dg_sampler_params;

/* The stop test of a round ([P1 四]).
 * DG_STOP_MEAN_ENTROPY: stop when this round's mean entropy < stop_threshold.
 * DG_STOP_TWO_ROUNDS: the page's adaptive stop.  Stop when this round's and
 *   the previous round's mean entropies are both < stop_threshold (0.005 on
 *   the page) and this round's argmax sequence equals the previous round's.
 *   The argmax is that of z = s*l/T in fp32 (ties -> lower index; for T == 0
 *   it is x_hat).  A round without a previous round (prev_* NULL) does not
 *   stop.
 * stop_threshold < 0 disables either test. */
enum { DG_STOP_MEAN_ENTROPY = 0, DG_STOP_TWO_ROUNDS = 1 };

/* Which positions a step keeps ([P1 四]).
 * DG_KEEP_TOPK: the keep_k positions of highest pmax (ties -> lower index).
 * DG_KEEP_ENTROPY_BUDGET: the page's entropy-ordered locking.  Positions are
 *   taken by increasing entropy (ties -> lower index); the first is always
 *   kept, and each later one while the running sum of entropies, the
 *   position itself included, is <= entropy_budget; the first position that
 *   crosses it and every later one are re-noised.  keep_k is ignored.  The
 *   sum is taken in fp64 over the fp32 per-position entropies. */
enum { DG_KEEP_TOPK = 0, DG_KEEP_ENTROPY_BUDGET = 1 };

/* Outputs of one sampler step; every pointer may be NULL (not written). */
typedef struct dg_step_out {
  int32_t* x_hat;            /* [B, N] sampled tokens */
  float* pmax;               /* [B, N] max probability of z */
  float* entropy;            /* [B, N] entropy of z, nats */
  int32_t* keep;             /* [B, N] 1 = kept, 0 = re-noised */
  float* mean_entropy;       /* [B] */
  int32_t* stop;             /* [B] 1 = stop test passed */
  int32_t* experts_touched;  /* [n_layers] distinct experts routed to */
  int32_t* argmax;           /* [B, N] argmax of z (ties -> lower index); pass it as the next
                                round's prev_argmax for DG_STOP_TWO_ROUNDS */
} dg_step_out;

/* A record of one layer of a forward pass, for layer-wise checks.  Rows are
 * the pass's B*N canvas positions in batch order (row b*N + i). */
typedef struct dg_layer_dump {
  int layer;             /* layer index, 0 .. n_layers-1 */
  float* hidden_in;      /* [B*N, d] fp32 residual stream entering the layer, or NULL */
  float* hidden_out;     /* [B*N, d] fp32 residual stream leaving it (after the MoE residual), or NULL */
  int32_t* expert_ids;   /* [B*N, k] the router's experts in this layer, selection order, or NULL */
  float* expert_wts;     /* [B*N, k] their softmax weights, or NULL */
} dg_layer_dump;

/* One denoising step ([P1 一/二/四]). */
typedef struct dg_step_args {
  int batch;                   /* B <= max_batch */
  const int* req;              /* HOST [B] request slots, distinct */
  int32_t* canvas;             /* [B, N] in: current canvas, out: re-noised canvas */
  const int32_t* prev_pred;    /* [B, N] previous x_hat for self-conditioning, or NULL */
  int step;                    /* t >= 1, Philox counter word 1 */
  dg_sampler_params sp;
  float* logits_out;           /* [B, N, V] fp32 to receive the logits (16-byte aligned), or NULL */
  float* hidden_out;           /* [B*N, d] fp32 residual stream before the final
                                  norm, or NULL */
  const dg_layer_dump* dump;   /* HOST pointer: record one layer of this pass, or NULL */
} dg_step_args;

/* One block ([P1 一/四], [P2], [P3]). */
typedef struct dg_block_args {
  int batch;                  /* B <= max_batch */
  const int* req;             /* HOST [B] request slots, distinct */
  int max_steps;              /* step budget (48 in [P1 四]) */
  int schedule_steps;         /* T of the keep schedule k_t = ceil(N t / T) */
  float temperature;
  float logit_scale_growth;   /* s_t = growth^(t-1) */
  float stop_threshold;       /* < 0 disables the adaptive stop */
  uint64_t seed;
  uint32_t block;
  int keep_mode;              /* DG_KEEP_TOPK (schedule k_t) or DG_KEEP_ENTROPY_BUDGET */
  float entropy_budget;       /* nats, for DG_KEEP_ENTROPY_BUDGET */
  int anneal;                 /* nonzero: linear temperature anneal ([P1 四]) */
  float temperature_end;      /* with anneal: step t runs at
                                 T_t = T + (T_end - T) (t-1) / (max_steps-1)
                                 (in double, then rounded to float; T_end when
                                 max_steps == 1).  Both ends > 0. */
  int stop_mode;              /* DG_STOP_MEAN_ENTROPY or DG_STOP_TWO_ROUNDS (the loop keeps
                                 the previous round's argmax and mean entropy) */
} dg_block_args;

/* Kernel-class timing, filled when profiling is on. */
typedef struct dg_profile_entry {
  const char* name;   /* static string */
  int launches;
  double ms;          /* summed CUDA-event time on the handle's stream */
} dg_profile_entry;

/*
 * dg_create: validate cfg, borrow w, allocate the KV cache
 * ([layers][max_batch][Hkv][max_ctx][hd] for K and the transposed
 * [layers][max_batch][Hkv][hd][max_ctx] for V, zero-filled) and the workspaces,
 * and build the TMA descriptors.  stream: a cudaStream_t (NULL = legacy default).
 * For n_layers == 0, w may be NULL (sampler-only handle for dg_sample).
 * BF16 handles need d, hd, F multiples of 64 and weight pointers 16-byte aligned.
 */
int dg_create(const dg_config* cfg, const dg_weights* w, void* stream, dg_handle** out);

/* Release everything the handle owns.  NULL is a no-op. */
void dg_destroy(dg_handle* h);

/* Message of the last failed call on h (NULL h: last failed dg_create). */
const char* dg_last_error(const dg_handle* h);

/*
 * Causal encode of n tokens per request at positions P..P+n-1, appending their
 * K/V to each request's cache (prompt prefill, [P1 二], [P2 架构基础]); then
 * P += n.  tokens: [B, n] int32.  DG_ECAPACITY if any P + n > max_ctx.
 */
int dg_prefill_prompt(dg_handle* h, int batch, const int* req, const int32_t* tokens, int n);

/*
 * Test hook: write positions [0, n) of one layer's cache for request req.
 * k, v: [Hkv, n, hd] in the handle's dtype.  Does not change P.
 */
int dg_set_kv(dg_handle* h, int req, int layer, const void* k, const void* v, int n);

/*
 * Test hook: read positions [0, n) of one layer's cache for request req into
 * k, v: [Hkv, n, hd] in the handle's dtype (K as RoPE'd, V as projected).
 * Does not change P.  DG_ECAPACITY if n > max_ctx.
 */
int dg_get_kv(dg_handle* h, int req, int layer, void* k, void* v, int n);

/* Set / read a request's cache length P (host-side state; set checks capacity). */
int dg_set_length(dg_handle* h, int req, int length);
int dg_get_length(const dg_handle* h, int req, int* length);

/*
 * One denoising step over B canvases: embed + self-conditioning, all layers
 * (canvas attention over cache [0,P) + the canvas, no mask), final norm, tied
 * LM head, then the sampler (dg_sample's definition).  The canvas K/V are
 * written at cache positions [P, P+N) as scratch; P is not changed.
 * DG_ECAPACITY if P + N > max_ctx.
 */
int dg_denoise_step(dg_handle* h, const dg_step_args* a, const dg_step_out* o);

/*
 * The sampler alone on caller logits [B, N, V] fp32 ([P1 四], [P1 五]):
 * z = s*l/T; pmax = max softmax(z); H = entropy(softmax(z));
 * x_hat = inverse-CDF sample in vocabulary order with u from Philox word 0 of
 * counter (i, step, block, req[b]) under key seed (u = (w0 >> 8) * 2^-24);
 * keep = top keep_k positions by pmax (ties to the lower index), or the
 * entropy-budget set when sp->keep_mode is DG_KEEP_ENTROPY_BUDGET;
 * canvas[b,i] = keep ? x_hat : (w1 * V) >> 32 (uniform re-noise from word 1);
 * mean entropy and stop = mean < stop_threshold.
 * logits must be 16-byte aligned (DG_EINVAL otherwise); an unknown keep_mode
 * or stop_mode, or a negative or non-finite entropy_budget, is DG_EINVAL.
 * With DG_STOP_TWO_ROUNDS the stop follows that mode's definition, and o->argmax
 * is required (DG_EINVAL without it): pass it back as the next round's
 * prev_argmax.  dg_denoise_step follows the same rule.
 */
int dg_sample(dg_handle* h, const float* logits, int batch, const int* req, int step,
              const dg_sampler_params* sp, int32_t* canvas, const dg_step_out* o);

/*
 * dg_sample without a handle and without allocating.  The pages have no
 * counterpart: this is a library convenience, not a step of the method.
 *
 * It computes exactly what dg_sample computes (same kernels, same Philox
 * counters) for logits [batch, n, vocab] fp32 (16-byte aligned).  It is meant
 * for callers that must not allocate device memory: a serving runtime that
 * reserved the GPU's memory up front, or code sampling from logits it already
 * owns.  Those callers cannot pay for dg_create, which allocates a KV cache and
 * workspaces.  This call never calls cudaMalloc, cudaFree or any allocating
 * library.  Its scratch is one fixed 8 MiB device array per device that the
 * CUDA runtime sets aside when this library's module loads.
 *
 * Arguments:
 *   req: HOST [batch] request ids (Philox counter word 3), each >= 0;
 *        1 <= batch <= 64.
 *   n: canvas length, 1..1024.
 *   step, sp: as for dg_sample; sp->keep_k <= n.
 *   canvas: device [batch, n]; in: unused, out: the re-noised canvas.
 *   o: as for dg_sample, or NULL.  x_hat / pmax / entropy that o does not
 *      request are kept in the scratch; experts_touched is ignored.
 *   stream: a cudaStream_t of the current device (NULL = legacy default).
 *   err: buffer of err_len bytes for a message (may be NULL).
 *
 * Limits and behaviour:
 *   - The request must fit the scratch:
 *     ceil(vocab / 4096) * 24 bytes per row of logits, plus ~16 bytes per row
 *     and 1.3 KB.  At vocab = 262144 that is about 5400 rows (21 canvases of 256).
 *     A larger request returns DG_ECAPACITY before anything is launched.
 *   - The first call on a device does the setup (looks up the scratch's
 *     address, loading the module if needed); make it before any stream capture.
 *   - Nothing in the scratch has to start at zero: a call reads only what it
 *     wrote itself.
 *   - Every call on a device shares the one scratch.  Calls on a device must
 *     therefore be ordered: the same stream, or streams ordered by events.
 *     Overlapping calls race on the scratch and give wrong results.
 *   - The request ids travel to the device as a kernel argument: the call
 *     makes no host-to-device copy and does not wait for the stream.
 *   - DG_STOP_TWO_ROUNDS needs o->argmax (DG_EINVAL without it): that row is
 *     the next round's prev_argmax, which the shared scratch cannot keep.
 *   - Returns DG_OK, DG_EINVAL (bad argument), DG_ECAPACITY (too large) or
 *     DG_ECUDA (a launch or runtime call failed).
 */
int dg_sample_noalloc(const float* logits, int batch, int n, int vocab, const int* req, int step,
                      const dg_sampler_params* sp, int32_t* canvas, const dg_step_out* o, void* stream,
                      char* err, size_t err_len);

/*
 * One block per request: canvas from Philox word 1 of counter (i, 0, block,
 * req); steps t = 1..max_steps with keep_k = ceil(N t / schedule_steps) (or
 * the entropy budget, per keep_mode), logit scale growth^(t-1), temperature T
 * or the annealed T_t, self-conditioning on the previous x_hat; a request
 * finishes at its first stop (or at max_steps) with output x_hat; the loop ends
 * when every request has finished.  Then the causal hand-off: the output tokens
 * are encoded causally and their K/V appended (P += N) ([P2], [P3]).
 * out_tokens: [B, N] device int32.  steps_used: HOST int, steps run.
 * DG_EINVAL for an unknown keep_mode or stop_mode, a negative or non-finite
 * budget, or an anneal end that is not > 0 (when anneal is set, the start
 * must be > 0 too).
 */
int dg_generate_block(dg_handle* h, const dg_block_args* a, int32_t* out_tokens, int* steps_used);

/* dg_generate_block with HOST output: copies the [B, N] tokens to out_tokens_host. */
int dg_generate_block_host(dg_handle* h, const dg_block_args* a, int32_t* out_tokens_host,
                           int* steps_used);

/*
 * AR mode ([P1 七]: the same weights load as an autoregressive model; [P1 五]
 * compares the canvas step with one AR step).  For each request: encode
 * tokens[b] causally at position P (its K/V appended, P += 1), then write the
 * logits of the token that follows it: final norm and tied LM head.  No canvas
 * and no self-conditioning.
 *   tokens: [B] device int32 in [0, V) (out-of-range tokens are replaced by 0
 *           and reported as DG_EINVAL by the next synchronising call).
 *   logits: [B, V] device fp32, 16-byte aligned.
 *   next_token: [B] device int32, the argmax of the logits (ties -> lower
 *           index), or NULL.
 * bf16 handles with head_dim 256 run the single-token attention kernel (one
 * pass over the cache per KV head, all its query heads together).
 * DG_ECAPACITY if any P + 1 > max_ctx.
 */
int dg_ar_step(dg_handle* h, int batch, const int* req, const int32_t* tokens, float* logits, int32_t* next_token);

/* Synchronise the handle's stream and report device-side timeouts. */
int dg_synchronize(dg_handle* h);

/* Kernel launches issued by this handle since creation. */
uint64_t dg_launch_count(const dg_handle* h);

/* Kernel classes of the profiler; bit k of dg_profile_enable's mask selects class k. */
enum {
  DG_PROF_EMBED = 0,
  DG_PROF_DENSE_GEMM = 1,     /* self-conditioning, QKV and O projections */
  DG_PROF_ROPE_SCATTER = 2,
  DG_PROF_ATTENTION = 3,      /* attention + split-KV combine */
  DG_PROF_RMSNORM = 4,
  DG_PROF_ROUTER = 5,         /* router logits, top-k, permutation */
  DG_PROF_GATHER = 6,
  DG_PROF_MOE_UP = 7,         /* grouped gate/up + SwiGLU */
  DG_PROF_MOE_DOWN = 8,
  DG_PROF_COMBINE = 9,
  DG_PROF_LM_HEAD = 10,
  DG_PROF_SAMPLER_ROWS = 11,
  DG_PROF_SAMPLER_FINISH = 12,
  DG_PROF_COUNT = 13
};
#define DG_PROFILE_ALL (-1)

/*
 * Per-kernel-class CUDA-event timing on the handle's stream.  mask = 0 turns
 * it off; otherwise bit k times class k (DG_PROFILE_ALL: every class).  Each
 * timed launch group costs two event records, so time only the classes you
 * read when the surrounding run is itself being timed.  dg_profile_read
 * synchronises; dg_profile_reset drops the records.
 */
int dg_profile_enable(dg_handle* h, int mask);
int dg_profile_read(dg_handle* h, dg_profile_entry* out, int max_entries, int* n_entries);
int dg_profile_reset(dg_handle* h);

/*
 * Test hook: Philox4x32-10 [Philox] on n counters.  ctr [n,4], key [n,2],
 * out [n,4] (this library's generator), out_curand [n,4] (cuRAND's device
 * Philox4_32_10 for the same key/counter, or NULL).  All device uint32.
 * Uses the handle's stream; h may be a sampler-only handle.
 */
int dg_selftest_philox(dg_handle* h, const uint32_t* ctr, const uint32_t* key, uint32_t* out,
                       uint32_t* out_curand, int n);

/*
 * Test hook: one dense bf16 GEMM through the tensor-core path,
 * out[T, M] (fp32) = x[T, K] * w[M, K]^T.  x, w bf16 row-major, 16-byte aligned,
 * K a multiple of 64.  Requires a bf16 handle (its stream and SM count are used).
 */
int dg_selftest_gemm(dg_handle* h, const void* x, const void* w, int T, int M, int K, float* out);

/*
 * Test hook: the split-K form the layers use for up to 256 tokens (QKV, O and
 * self-conditioning projections).  Writes *nsplit (<= max_split) fp32 partial
 * slices part[s][T][M], whose sum over s is x[T, K] * w[M, K]^T.  part holds
 * max_split * T * M floats.  Same operand rules as dg_selftest_gemm;
 * DG_EINVAL if T > 256.
 */
int dg_selftest_gemm_split(dg_handle* h, const void* x, const void* w, int T, int M, int K, float* part,
                           int max_split, int* nsplit);

/*
 * Test hook: the same split-K product on CTA pairs (two SMs compute one
 * 256-row weight tile, each loading 128 weight rows and half of the token
 * tile).  ksplit fp32 slices part[s][T][M] sum to x[T, K] * w[M, K]^T; ntile
 * (token rows of a pair's tile) is 64, 128 or 256 and ksplit is in
 * [1, K / 64].  Same operand rules as dg_selftest_gemm; DG_EINVAL otherwise.
 */
int dg_selftest_gemm_pair(dg_handle* h, const void* x, const void* w, int T, int M, int K, int ntile, int ksplit,
                          float* part);

/*
 * Test hook for the bounded device waits: one kernel waits on a shared-memory
 * barrier that nothing arrives on, gives up after limit_us microseconds of wall
 * time (1 .. 100000), records the timeout and returns.  The call synchronises
 * and returns what any synchronising call then reports: DG_ETIMEOUT, with the
 * device error flag cleared, so the handle stays usable.
 */
int dg_selftest_wait_timeout(dg_handle* h, int limit_us);

/*
 * NVFP4 quantisation of n_mats bf16 matrices w [n_mats][rows][K] (K a multiple
 * of 64, rows >= 1), the storage of DG_EXPERT_NVFP4, computed on the device
 * without allocating.  Per matrix: g = fp32(amax / (6 * 448)) (1 for an
 * all-zero matrix); per block of 16 elements of a row: scale code
 * s = E4M3(amax_b / (6 g)); element code q = E2M1(w / (E4M3(s) g)), both
 * rounded to nearest with ties to the even code and saturated (a block whose
 * scale is 0 gets codes 0).  Quotients are formed in fp64.
 *   codes:  [n_mats][rows][K/2] bytes (element 2j in the low nibble)
 *   scales: [n_mats][K/64][rows_pad][4] bytes, rows_pad = rows rounded up to
 *           128; padding rows are written as 0
 *   g:      [n_mats] fp32
 * All device pointers; stream: a cudaStream_t (NULL = legacy default).
 * Returns DG_OK, DG_EINVAL (bad shape, null or unaligned pointer: w and codes
 * 16-byte aligned) or DG_ECUDA; err (err_len bytes, may be NULL) gets the message.
 */
int dg_quantize_nvfp4(const void* w, int n_mats, int rows, int K, uint8_t* codes, uint8_t* scales, float* g,
                      void* stream, char* err, size_t err_len);

/* Outputs of the router self-test (all device pointers, all required). */
typedef struct dg_router_out {
  int32_t* ids;      /* [T, k] selected experts, in selection order (logit desc, id asc) */
  float* wts;        /* [T, k] softmax of the k selected biased logits */
  int32_t* cnt;      /* [E] items routed to each expert */
  int32_t* off;      /* [E + 1] exclusive prefix sum of cnt */
  int32_t* perm;     /* [T * k] item t*k+s at position off[e] + (its rank among expert e's items, by item index) */
  int32_t* work;     /* [3 * (E + ceil(T * k / tile))] (expert, first position, rows <= tile) tiles, experts
                        ascending */
  int32_t* n_work;   /* [1] number of work tiles */
  int32_t* touched;  /* [1] number of experts with cnt > 0 */
} dg_router_out;

/*
 * Test hook: the router of one layer ([P1 二]: 128 experts, 8 per token) run
 * by the kernels the layers use, on caller logits.  logits [T, E] fp32 (the
 * gate projection x W_r^T), bias [E] fp32 or NULL, both 16-byte aligned for the
 * vector form (any alignment works).  g = logits + bias; top-k by g with ties
 * to the lower id (no expert twice, -inf included); softmax over the k
 * selected; then the counting sort into expert order, the work list and the
 * distinct-expert count.  E <= 256, k <= min(E, 16), 1 <= tile <= 1024.
 * Uses the handle's stream; h may be a sampler-only handle.
 */
int dg_selftest_router(dg_handle* h, const float* logits, const float* bias, int T, int E, int k, int tile,
                       const dg_router_out* o);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
