// Host-side launchers of the device kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

constexpr int kMaxBatch = 64;

// Per-launch description of the requests in a forward pass: row b of the
// batch is request slot `slot[b]` whose cache holds `len[b]` positions before
// this pass.
struct BatchInfo {
  int B;
  int slot[kMaxBatch];
  int len[kMaxBatch];
};

// ---- elementwise / small kernels (k_elementwise.cu)
// h[t,:] = E[tok[t],:] (fp32); if prev != null, eprev[t,:] = E[prev[t],:] (act dtype)
template <typename T>
void launch_embed(const int32_t* tok, const int32_t* prev, const T* embed, float* h, T* eprev, int n_tok,
                  int d, int vocab, int* err, cudaStream_t s);
// xn[t,:] = h[t,:] * w / sqrt(mean(h^2) + eps)
template <typename T>
void launch_rmsnorm(const float* h, const float* w, T* xn, int n_tok, int d, float eps, cudaStream_t s);
// h[t,:] += sum_s wts[t,s] * y[t*k+s,:] (slot order, fp32), then optional xn = rmsnorm(h, norm_w).
// y holds the expert outputs in the activation type T.
template <typename T>
void launch_combine(float* h, const T* y, const float* wts, int k, const float* norm_w, T* xn,
                    int n_tok, int d, float eps, cudaStream_t s);
// h[t,:] += sum over s < nsplit (in order) of part[s*split_stride + t*d + :]; then
// xn = rmsnorm(h, w).  Sums the K slices of a split-K projection into the residual.
template <typename T>
void launch_add_rmsnorm(float* h, const float* part, int nsplit, size_t split_stride, const float* w, T* xn,
                        int n_tok, int d, float eps, cudaStream_t s);
// Split fp32 q|k|v rows into rotated Q [B,Hq,nq,hd], K cache rows and transposed V cache rows.
// The rows are the sum of nsplit K slices qkv + s*split_stride (nsplit 1: qkv itself).
template <typename T>
void launch_rope_scatter(const float* qkv, int nsplit, size_t split_stride, T* q, T* kc, T* vt,
                         const float* rope_cs, const BatchInfo& bi, int nq, int hq, int hkv, int hd, int max_ctx,
                         cudaStream_t s);
// xp[p,:] = xn[perm[p]/k,:] for p < n_rows
template <typename T>
void launch_gather_rows(const T* xn, const int32_t* perm, T* xp, int n_rows, int k, int d, cudaStream_t s);
// canvas[b,i] = uniform token from Philox word 1 of counter (i, 0, block, req[b])
void launch_init_canvas(int32_t* canvas, const BatchInfo& bi, const int* req_ids, int n, int vocab,
                        uint64_t seed, uint32_t block, cudaStream_t s);
// Copy a [Hkv, n, hd] K/V block into positions [0, n) of one request's cache.
template <typename T>
void launch_set_kv(const T* k, const T* v, T* kc, T* vt, int hkv, int n, int hd, int max_ctx,
                   cudaStream_t s);

// Copy positions [0, n) of one request's cache out to [Hkv, n, hd] K/V blocks.
template <typename T>
void launch_get_kv(const T* kc, const T* vt, T* k, T* v, int hkv, int n, int hd, int max_ctx,
                   cudaStream_t s);
// One thread waits on an mbarrier nothing arrives on; records a timeout after limit_ns.
void launch_wait_timeout_selftest(int* err, unsigned long long limit_ns, cudaStream_t s);

// ---- router (k_router.cu)
// Per token: g = glog + bias; top-k (ties -> lower id); softmax over the k.
// glog holds nsplit partial-sum slices of [n_tok, e] at a stride of n_tok*e
// floats; they are added in slice order.
void launch_router_topk(const float* glog, int nsplit, const float* bias, int32_t* ids, float* wts, int n_tok,
                        int e, int k, cudaStream_t s);
// Deterministic counting sort of the n_tok*k (token, slot) items by expert
// (tokens ascending inside an expert).  perm[pos] = t*k+s; cnt[E]; off[E+1];
// work list of (expert, first row, rows) tiles of at most `tile` rows;
// touched = number of experts with cnt > 0.
void launch_router_permute(const int32_t* ids, int n_items, int e, int tile, int32_t* cnt, int32_t* off,
                           int32_t* perm, int32_t* work, int32_t* n_work, int32_t* touched,
                           cudaStream_t s);

// Sampler statistics of one token over one group of 32 consecutive vocabulary
// entries, z = logit * scale: the group max, the first index holding it, and
// sum exp(z - m), sum exp(z - m)(z - m) (fp32 over the 32 terms).  In arg-max
// mode (temperature 0) s counts the entries equal to m and a is 0.
struct VocabStat {
  float m;
  int idx;
  float s;
  float a;
};

// ---- sampler (k_sampler.cu)
struct SamplerArgs {
  float temperature, logit_scale, stop_threshold;
  int keep_k;
  uint64_t seed;
  uint32_t block;
  uint32_t step;
  int keep_mode = 0;            // 0: top keep_k by pmax; 1: entropy budget
  float entropy_budget = 0.f;   // nats, keep_mode 1
  int stop_mode = 0;            // 0: mean entropy; 1: two rounds (mean entropies and argmax)
  const int32_t* prev_argmax = nullptr;   // stop_mode 1: previous round [B, N], or null
  const float* prev_mean_h = nullptr;     // stop_mode 1: previous round [B], or null
};
size_t sampler_workspace_bytes(int rows, int vocab);
// rows = B*N logits rows; writes x_hat, pmax, H (workspace-sized arrays) and,
// when argmax is not null, the argmax of z per row (ties -> lower index).
void launch_sampler_rows(const float* logits, int rows, int n, int vocab, const int* req_ids,
                         const SamplerArgs& a, void* ws, int32_t* x_hat, float* pmax, float* ent,
                         cudaStream_t s, int32_t* argmax = nullptr);
// The sampler rows from the LM head's per-group statistics instead of logits:
// merges each row's n_groups VocabStat records in vocabulary order (fp64), draws
// the Philox inverse-CDF sample, and recomputes only the 32 logits of the group
// holding u*S from the final-norm rows xn [rows, d] and the tied embedding
// [V, d] (bf16).  Same outputs as launch_sampler_rows.
void launch_sampler_fused_rows(const VocabStat* stats, int n_groups, const __nv_bfloat16* xn,
                               const __nv_bfloat16* embed, int d, int rows, int n, int vocab, const int* req_ids,
                               const SamplerArgs& a, int32_t* x_hat, float* pmax, float* ent, cudaStream_t s,
                               int32_t* argmax = nullptr);
// Per canvas: keep set, re-noise, mean entropy, stop; optional block-loop outputs.
// argmax: this round's argmax rows (required by stop_mode 1).
void launch_sampler_finish(const int32_t* x_hat, const float* pmax, const float* ent, int B, int n,
                           int vocab, const int* req_ids, const SamplerArgs& a, int32_t* canvas,
                           int32_t* keep, float* mean_h, int32_t* stop, int32_t* done, int32_t* out_tokens,
                           int final_step, cudaStream_t s, const int32_t* argmax = nullptr);

// ---- GEMMs
enum Epi { EPI_STORE_F32 = 0, EPI_ADD_F32 = 1, EPI_STORE_ACT = 2, EPI_SWIGLU_ACT = 3, EPI_SCATTER_ACT = 4,
           EPI_VOCAB_STATS = 5 };


// SIMT fp32/generic path: out[t, n] (op)= sum_k x[t,k] w[n,k].
template <typename T>
void launch_gemm_simt(const T* x, const T* w, int n_tok, int n_out, int kdim, Epi epi, void* out, int ld_out,
                      const float* bias, cudaStream_t s);
// SIMT grouped expert GEMM over a work list (expert, row0, rows):
// up:   out[r, f]  = silu(x[r] . wg[e,f]) * (x[r] . wu[e,f])      (act dtype)
// down: y[perm[r], n] = x[r] . wd[e,n]                              (fp32)
template <typename T>
void launch_grouped_simt(const T* x, const T* wa, const T* wb, int n_out, int kdim, const int32_t* work,
                         const int32_t* n_work, int n_work_max, const int32_t* perm, bool up, void* out,
                         int ld_out, cudaStream_t s);

// tcgen05 path (k_gemm_tc.cu): weights are the 128-row M side, tokens the N side.
struct TcGemm {
  int mode;          // 0 dense, 1 grouped up (gate+up, SwiGLU), 2 grouped down
  int M, K;          // weight rows (dense: total; grouped: per expert), reduction dim
  int T;             // dense: token rows
  int ntile;         // token tile width (multiple of 32, <= 256)
  int seg1, seg2;    // dense: first weight row served by map a1 / a2 (multiples of 128)
  const int32_t* work;
  const int32_t* n_work;
  int n_work_max;
  int epi;
  void* out;
  int ld_out;
  const float* bias;
  const int32_t* row_map;
  int* err;
  int ksub;          // 64-wide K blocks per pipeline stage (0 = build default)
  int ctas_per_sm;   // co-resident CTAs the grid is sized for (0 = build default)
  int ksplit;        // dense EPI_STORE_F32 only: K split into ksplit slices, slice s
                     // writes its partial sums at out + s * split_stride (floats)
  size_t split_stride;
  int tma_out;       // set by the launcher: the output goes out through TMA stores
  // EPI_VOCAB_STATS (dense, the tied LM head): out is VocabStat [T][n_groups] with
  // n_groups = ceil(M / 32); the logits are scaled by zscale (argmax_mode: counts of maxima)
  float zscale;
  int argmax_mode;
  int n_groups;
};
// Returns 0, or -1 when the tile does not fit a two-stage pipeline (nothing launched).
// b: token map with boxes of ntile rows.  bsub (grouped modes, or NULL): maps of the
// same tokens with boxes of 32, 64, 128 rows (those below ntile), used for work
// items with fewer rows.
// tout (dense EPI_STORE_F32, or NULL): fp32 map of the output as (M, T, ksplit) with boxes of
// (128, 32, 1); the epilogue then writes each 32-row chunk with one TMA store.
int launch_gemm_tc(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b,
                   const CUtensorMap* bsub, const TcGemm& p, int num_sms, cudaStream_t s,
                   const CUtensorMap* tout = nullptr);
int gemm_tc_smem_bytes(const TcGemm& p, int* stages);
// Dense mode (EPI_STORE_F32, split-K slices as launch_gemm_tc) on CTA pairs
// (k_gemm_tc2.cu): 256-row weight tiles, each CTA of a pair holding 128 weight
// rows and half of the token tile.  a0..a2: weight maps with boxes of 128 rows
// by g.ksub (1, 2 or 4) 64-column chunks; b: token map with boxes of ntile/2
// rows by g.ksub chunks;
// tout: fp32 output map as for launch_gemm_tc, or NULL.  seg1 / seg2 must be
// multiples of 256.  Returns -1 (nothing launched) for another shape.
int launch_gemm_tc_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b,
                        const TcGemm& g, int num_sms, cudaStream_t s, const CUtensorMap* tout);

// Grouped modes 1 (gate/up + SwiGLU) and 2 (down + scatter) on CTA pairs
// (k_moe_tc2.cu): 256-row weight blocks, each CTA of a pair holding 128 weight
// rows and half of the item's token rows.  a0 / a1: expert weight maps (64,
// rows, K/64, E) with boxes of 128 rows x g.ksub chunks (a1: the up weights,
// mode 1); b16 / b32 / b64 / b128: token maps with boxes of 16 / 32 / 64 /
// 128 rows x g.ksub chunks (b128 is read only when g.ntile > 128).  Work items
// of up to 256 rows (g.ntile <= 256).  Returns -1 (nothing launched) for
// another shape.
int launch_gemm_tc2_grouped(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b16,
                            const CUtensorMap& b32, const CUtensorMap& b64, const CUtensorMap& b128, const TcGemm& g,
                            int num_sms, cudaStream_t s);

// NVFP4 grouped expert GEMMs (k_gemm_fp4.cu): modes 1 (gate/up + SwiGLU) and 2
// (down + scatter) of the bf16 grouped GEMM, with the weights as E2M1 codes
// (c0 / c1: uint8 maps (K/2 bytes, M rows, E) with boxes of 32 bytes x 128
// rows), tiled E4M3 scales and per-expert fp32 scales.  b / bsub: the token
// maps, as for launch_gemm_tc.  Returns -1 (nothing launched) for an
// unsupported shape.
struct Fp4Gemm {
  int mode;
  int M, K;
  int ntile;
  const int32_t* work;
  const int32_t* n_work;
  int n_work_max;
  void* out;
  int ld_out;
  const int32_t* row_map;
  int* err;
  const uint8_t* sf0;
  const uint8_t* sf1;
  const float* g0;
  const float* g1;
};
int launch_gemm_fp4(const CUtensorMap& c0, const CUtensorMap& c1, const CUtensorMap& b, const CUtensorMap* bsub,
                    const Fp4Gemm& g, int num_sms, cudaStream_t s);

// ---- attention
struct AttnArgs {
  int B, nq, hq, hkv, hd, max_ctx;
  int causal;
  BatchInfo bi;
};
// SIMT (any dtype): q [B,Hq,nq,hd]; kc [slots,Hkv,max_ctx,hd]; vt [slots,Hkv,hd,max_ctx];
// out [B*nq, Hq*hd]
template <typename T>
void launch_attn_simt(const T* q, const T* kc, const T* vt, T* out, const AttnArgs& a, cudaStream_t s);

// tcgen05 canvas/causal attention for bf16, hd == 256 (k_attn_tc.cu).
struct AttnTcArgs {
  AttnArgs a;
  int n_split;       // KV splits per (b, head, q-tile)
  float* part_o;     // [splits][B][Hq][nq_pad][hd] fp32 partial outputs (unnormalised)
  float* part_ml;    // [splits][B][Hq][nq_pad][2] (max, sum)
  int nq_pad;
  int* err;
};
void launch_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    __nv_bfloat16* out, const AttnTcArgs& a, cudaStream_t s);
size_t attn_tc_partial_floats(int n_split, int B, int hq, int nq_pad, int hd);
// The same on CTA pairs (k_attn_tc2.cu): query heads 2y and 2y+1 (one KV head)
// share every K/V byte, 128-key tiles.  tv: V^T map with boxes of 64 keys x
// 128 dims.  Needs hd == 256 and an even number of query heads per KV head
// (attn_tc2_supported).  Same partial layout and combine as launch_attn_tc.
// tpo (or NULL: plain stores): fp32 map over part_o as (256 columns, nq rows,
// n_split * B * Hq planes) with boxes of 32 x 128 x 1 and 128-byte swizzle.
bool attn_tc2_supported(int hq, int hkv, int hd);
void launch_attn_tc2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap* tpo,
                     __nv_bfloat16* out, const AttnTcArgs& a, cudaStream_t s);
// Merge KV-split partials (unnormalised O [split][B*Hq*nq][256], (max log2, sum)) into
// out [B*nq, Hq*256] bf16.
void launch_attn_combine(const float* part_o, const float* part_ml, __nv_bfloat16* out, int n_split, int B, int hq,
                         int nq, cudaStream_t s);
// Single-token attention (AR decode, k_attn_decode.cu): bf16, hd 256, nq 1, Hq/Hkv in {1,2,4,8};
// q [B][Hq][1][hd]; keys are the cache [0, len] of each request.  Split partials in
// part_o / part_ml (capacity part_rows_cap split rows), then the combine.  Returns -1
// (nothing launched) for another shape.
int launch_attn_decode(const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vt,
                       __nv_bfloat16* out, const AttnArgs& a, float* part_o, float* part_ml, size_t part_rows_cap,
                       int num_sms, cudaStream_t s);

// ---- self test
void launch_philox_selftest(const uint32_t* ctr, const uint32_t* key, uint32_t* out, uint32_t* out_curand,
                            int n, cudaStream_t s);

}  // namespace dg
