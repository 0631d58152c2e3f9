// The sampler ([P1 四]: confidence, entropy, keep the confident positions,
// re-randomise the rest, adaptive stop on mean entropy; [P1 五]: a softmax over
// the full ~262k vocabulary per canvas position).
//
// Pass 1 (HBM-bound): each CTA reduces one 4096-logit chunk of one row to
// (max, sum exp(z-max), sum exp(z-max)(z-max)) with 128-bit loads.
// Pass 2: one CTA per row merges the chunk partials in chunk order, derives
// pmax and the entropy, and draws the inverse-CDF sample: the chunk holding
// u*S is found from the partials and only that chunk is re-read and scanned
// in vocabulary order.
// Pass 3: one CTA per canvas ranks positions by pmax, keeps the top-k,
// re-noises the rest with Philox, and forms the mean entropy / stop flag.
// On request, passes 1 and 2 also carry the first arg-max of z per row, for
// the two-round stop.
#include <curand_kernel.h>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

constexpr int kChunk = 4096;
constexpr int kThreads = 256;
constexpr int kPerThread = kChunk / kThreads;  // 16

struct Partial {
  float m;    // chunk max of z (T > 0) / of the scaled logit (T == 0)
  int idx;    // first arg-max index in the chunk (T == 0, or when requested; else 0)
  double s;   // sum exp(z - m)             | T == 0: count of maxima
  double a;   // sum exp(z - m) * (z - m)
};

size_t sampler_workspace_bytes(int rows, int vocab) {
  const size_t n_chunks = (vocab + kChunk - 1) / kChunk;
  return (size_t)rows * n_chunks * sizeof(Partial);
}

__device__ __forceinline__ void load_chunk(const float* __restrict__ row, int c0, int vocab, float scale,
                                           float (&z)[kPerThread], bool vec4) {
  if (vec4) {
#pragma unroll
    for (int r = 0; r < kPerThread / 4; ++r) {
      const int j = c0 + (threadIdx.x + r * kThreads) * 4;
      float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (j < vocab) v = __ldcs(reinterpret_cast<const float4*>(row + j));  // j+3 < vocab since vocab % 4 == 0
      z[4 * r + 0] = (j < vocab) ? v.x * scale : -INFINITY;
      z[4 * r + 1] = (j < vocab) ? v.y * scale : -INFINITY;
      z[4 * r + 2] = (j < vocab) ? v.z * scale : -INFINITY;
      z[4 * r + 3] = (j < vocab) ? v.w * scale : -INFINITY;
    }
  } else {
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
      const int j = c0 + threadIdx.x + r * kThreads;
      z[r] = (j < vocab) ? row[j] * scale : -INFINITY;
    }
  }
}

// vocabulary index of register r of this thread in the load pattern above
__device__ __forceinline__ int reg_index(int c0, int r, bool vec4) {
  return vec4 ? c0 + (threadIdx.x + (r >> 2) * kThreads) * 4 + (r & 3) : c0 + threadIdx.x + r * kThreads;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The exponentials are fp32 (expf); every sum over the vocabulary is carried
// in fp64 so the CDF that decides the sample is not limited by fp32 rounding
// of 262144-term sums.
__global__ void __launch_bounds__(kThreads) sampler_pass1(const float* __restrict__ logits, int vocab, float scale,
                                                          int argmax_mode, int want_idx, Partial* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red_m[kThreads / 32];
  __shared__ double red_s[kThreads / 32];
  __shared__ double red_a[kThreads / 32];
  __shared__ int red_i[kThreads / 32];
  __shared__ int red_c[kThreads / 32];
  const int c = blockIdx.x, row = blockIdx.y;
  const int n_chunks = gridDim.x;
  const int c0 = c * kChunk;
  const bool vec4 = (vocab % 4) == 0;
  float z[kPerThread];
  load_chunk(logits + (size_t)row * vocab, c0, vocab, scale, z, vec4);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < kPerThread; ++r) m = fmaxf(m, z[r]);
  m = warp_max(m);
  if (lane == 0) red_m[w] = m;
  __syncthreads();
  m = red_m[0];
#pragma unroll
  for (int x = 1; x < kThreads / 32; ++x) m = fmaxf(m, red_m[x]);
  Partial p;
  if (argmax_mode) {
    int idx = 0x7fffffff, cntm = 0;
#pragma unroll
    for (int r = 0; r < kPerThread; ++r)
      if (z[r] == m) { idx = min(idx, reg_index(c0, r, vec4)); ++cntm; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      idx = min(idx, __shfl_xor_sync(0xffffffffu, idx, o));
      cntm += __shfl_xor_sync(0xffffffffu, cntm, o);
    }
    if (lane == 0) { red_i[w] = idx; red_c[w] = cntm; }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int x = 1; x < kThreads / 32; ++x) { idx = min(idx, red_i[x]); cntm += red_c[x]; }
      p.m = m;
      p.idx = idx;
      p.s = (double)cntm;
      p.a = 0.0;
      part[(size_t)row * n_chunks + c] = p;
    }
    return;
  }
  int first = 0;
  if (want_idx) {  // uniform over the block
    int best = 0x7fffffff;
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
      const int j = reg_index(c0, r, vec4);
      if (z[r] == m && j < vocab) best = min(best, j);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) red_i[w] = best;
    __syncthreads();
    if (threadIdx.x == 0)
      for (int x = 0; x < kThreads / 32; ++x) best = min(best, red_i[x]);
    first = best;
  }
  double s = 0.0, a = 0.0;
  if (m > -INFINITY) {
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
      const float d = z[r] - m;
      const float e = expf(d);      // exp(-inf) = 0 for padding
      s += (double)e;
      a += (e > 0.f) ? (double)e * (double)d : 0.0;
    }
  }
  s = warp_sum_d(s);
  a = warp_sum_d(a);
  if (lane == 0) { red_s[w] = s; red_a[w] = a; }
  __syncthreads();
  if (threadIdx.x == 0) {
    s = 0.0; a = 0.0;
    for (int x = 0; x < kThreads / 32; ++x) { s += red_s[x]; a += red_a[x]; }
    p.m = m; p.idx = first; p.s = s; p.a = a;
    part[(size_t)row * n_chunks + c] = p;
  }
}

__global__ void __launch_bounds__(kThreads) sampler_pass2(const float* __restrict__ logits, int n, int vocab,
                                                          float scale, int argmax_mode, const int* __restrict__ req_ids,
                                                          uint64_t seed, uint32_t step, uint32_t block,
                                                          const Partial* __restrict__ part, int32_t* __restrict__ x_hat,
                                                          float* __restrict__ pmax, float* __restrict__ ent,
                                                          int32_t* __restrict__ argmax) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sh_M;
  __shared__ double sh_target, sh_P0;
  __shared__ int sh_c;
  __shared__ double scan[kThreads];
  __shared__ int sh_pick;
  __shared__ int sh_last;
  const int row = blockIdx.x;
  if (threadIdx.x == 0) sh_last = 0;
  const int b = row / n, i = row - b * n;
  const int n_chunks = (vocab + kChunk - 1) / kChunk;
  const Partial* pr = part + (size_t)row * n_chunks;
  if (argmax_mode) {
    if (threadIdx.x == 0) {
      float M = -INFINITY;
      for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, pr[c].m);
      int idx = -1;
      double cntm = 0.0;
      for (int c = 0; c < n_chunks; ++c)
        if (pr[c].m == M) {
          if (idx < 0) idx = pr[c].idx;
          cntm += pr[c].s;
        }
      x_hat[row] = idx;
      if (argmax) argmax[row] = idx;
      pmax[row] = (float)(1.0 / cntm);
      ent[row] = (float)log(cntm);
    }
    return;
  }
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, pr[c].m);
    if (argmax) {  // chunks are in vocabulary order: the first holding M has the first arg-max
      int idx = -1;
      for (int c = 0; c < n_chunks && idx < 0; ++c)
        if (pr[c].m == M) idx = pr[c].idx;
      argmax[row] = idx;
    }
    double S = 0.0, A = 0.0;
    for (int c = 0; c < n_chunks; ++c) {
      const double f = exp((double)pr[c].m - (double)M);
      S += pr[c].s * f;
      A += (pr[c].a + ((double)pr[c].m - (double)M) * pr[c].s) * f;
    }
    const Philox4 w = sampler_words(seed, (uint32_t)i, step, block, (uint32_t)req_ids[b]);
    const double target = (double)unit_uniform(w.w[0]) * S;
    // first chunk whose inclusive prefix exceeds the target (chunk order)
    double P = 0.0, P0 = 0.0;
    int cs = -1, last_pos = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const double sc = pr[c].s * exp((double)pr[c].m - (double)M);
      if (sc > 0.0) last_pos = c;
      if (cs < 0 && P + sc > target) { cs = c; P0 = P; }
      P += sc;
    }
    if (cs < 0) { cs = last_pos; P0 = INFINITY; }  // rounding: no crossing -> last positive
    sh_M = M; sh_target = target; sh_P0 = P0; sh_c = cs;
    pmax[row] = (float)(1.0 / S);
    ent[row] = (float)(log(S) - A / S);
  }
  __syncthreads();
  // scan chunk sh_c in vocabulary order: thread t owns 16 consecutive elements
  const float M = sh_M;
  const double target = sh_target, P0 = sh_P0;
  const int c0 = sh_c * kChunk;
  const float* lrow = logits + (size_t)row * vocab;
  float e[kPerThread];
  double local = 0.0;
  int lastpos = -1;
#pragma unroll
  for (int r = 0; r < kPerThread; ++r) {
    const int j = c0 + threadIdx.x * kPerThread + r;
    const float v = (j < vocab) ? expf(lrow[j] * scale - M) : 0.f;
    e[r] = v;
    local += (double)v;
    if (v > 0.f) lastpos = j;
  }
  // inclusive scan of the per-thread sums in thread order (Hillis-Steele)
  scan[threadIdx.x] = local;
  __syncthreads();
  for (int o = 1; o < kThreads; o <<= 1) {
    const double add = (threadIdx.x >= o) ? scan[threadIdx.x - o] : 0.0;
    __syncthreads();
    scan[threadIdx.x] += add;
    __syncthreads();
  }
  if (threadIdx.x == 0) sh_pick = 0x7fffffff;
  __syncthreads();
  const double before = P0 + (scan[threadIdx.x] - local);
  if (before <= target && before + local > target) {
    double run = before;
    int pick = -1;
#pragma unroll
    for (int r = 0; r < kPerThread; ++r) {
      run += (double)e[r];
      if (pick < 0 && run > target) pick = c0 + threadIdx.x * kPerThread + r;
    }
    if (pick < 0) pick = lastpos;  // the thread sum crossed but the element walk fell short
    atomicMin(&sh_pick, pick);
  }
  __syncthreads();
  if (sh_pick == 0x7fffffff) {
    // no crossing in this chunk (rounding): the last element with e > 0
    if (lastpos >= 0) atomicMax(&sh_last, lastpos);
    __syncthreads();
    if (threadIdx.x == 0) x_hat[row] = sh_last;
    return;
  }
  if (threadIdx.x == 0) x_hat[row] = sh_pick;
}

void launch_sampler_rows(const float* logits, int rows, int n, int vocab, const int* req_ids, const SamplerArgs& a,
                         void* ws, int32_t* x_hat, float* pmax, float* ent, cudaStream_t s, int32_t* argmax) {
  if (rows <= 0) return;
  const int n_chunks = (vocab + kChunk - 1) / kChunk;
  const int argmax_mode = a.temperature == 0.f;
  const float scale = argmax_mode ? a.logit_scale : a.logit_scale / a.temperature;
  Partial* part = reinterpret_cast<Partial*>(ws);
  const int want_idx = (argmax != nullptr && !argmax_mode) ? 1 : 0;
  launch_k(sampler_pass1, dim3(dim3(n_chunks, rows)), dim3(kThreads), 0, s, logits, vocab, scale, argmax_mode, want_idx,
           part);
  launch_k(sampler_pass2, dim3(rows), dim3(kThreads), 0, s, logits, n, vocab, scale, argmax_mode, req_ids, a.seed, a.step, a.block,
                                          part, x_hat, pmax, ent, argmax);
}

// Pass 2 on the LM head's per-group statistics (the fused form): one CTA per
// row.  Thread t merges groups [t*per, (t+1)*per) in order (fp64), the block
// merges the threads in order: the max M and its first index, S = sum of the
// group masses s_g exp(m_g - M), and the entropy term.  The inclusive scan of
// the threads' masses finds the thread, then the group, whose prefix first
// exceeds u*S; only that group's 32 logits are recomputed (the final-norm row
// times 32 embedding rows, fp32 accumulation) and walked in vocabulary order.
// The recomputed logits can differ from the GEMM's in the last bits, so a
// crossing that falls short inside the group takes the group's last positive
// entry, as a crossing that falls short anywhere does.
constexpr int kFusedThreads = 256;
constexpr int kGroup = 32;

__global__ void __launch_bounds__(kFusedThreads)
    sampler_pass2_fused(const VocabStat* __restrict__ st, int n_groups, const __nv_bfloat16* __restrict__ xn,
                        const __nv_bfloat16* __restrict__ emb, int d, int n, int vocab, float scale, int argmax_mode,
                        const int* __restrict__ req_ids, uint64_t seed, uint32_t step, uint32_t block,
                        int32_t* __restrict__ x_hat, float* __restrict__ pmax, float* __restrict__ ent,
                        int32_t* __restrict__ argmax) {
  pdl_wait();
  pdl_trigger();
  __shared__ double scan[kFusedThreads];
  __shared__ double red_a[kFusedThreads / 32];
  __shared__ float red_m[kFusedThreads / 32];
  __shared__ int red_i[kFusedThreads / 32];
  __shared__ int red_l[kFusedThreads / 32];
  __shared__ float sh_z[kGroup];
  __shared__ int sh_g;
  __shared__ double sh_P0;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int b = row / n, i = row - b * n;
  const VocabStat* pr = st + (size_t)row * n_groups;
  const int per = (n_groups + kFusedThreads - 1) / kFusedThreads;
  const int g0 = min(n_groups, tid * per), g1 = min(n_groups, g0 + per);
  // the max and its first index (groups in vocabulary order: strict > keeps the earlier one)
  float Mt = -INFINITY;
  int It = 0x7fffffff;
  for (int g = g0; g < g1; ++g) {
    const float m = pr[g].m;
    if (m > Mt) { Mt = m; It = pr[g].idx; }
  }
  float M = warp_max(Mt);
  if (lane == 0) red_m[w] = M;
  __syncthreads();
  M = red_m[0];
  for (int x = 1; x < kFusedThreads / 32; ++x) M = fmaxf(M, red_m[x]);
  int I = Mt == M ? It : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) I = min(I, __shfl_xor_sync(0xffffffffu, I, o));
  if (lane == 0) red_i[w] = I;
  // this thread's mass (relative to M), entropy term and last group with mass, in group order
  double wt = 0.0, at = 0.0;
  int lastg = -1;
  for (int g = g0; g < g1; ++g) {
    const VocabStat p = pr[g];
    if (argmax_mode) {
      if (p.m == M) wt += (double)p.s;
    } else {
      const double f = exp((double)p.m - (double)M);
      const double c = (double)p.s * f;
      wt += c;
      at += ((double)p.a + ((double)p.m - (double)M) * (double)p.s) * f;
      if (c > 0.0) lastg = g;
    }
  }
  int L = lastg;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L = max(L, __shfl_xor_sync(0xffffffffu, L, o));
  double a_w = warp_sum_d(at);
  if (lane == 0) { red_a[w] = a_w; red_l[w] = L; }
  scan[tid] = wt;
  __syncthreads();
  I = red_i[0];
  for (int x = 1; x < kFusedThreads / 32; ++x) I = min(I, red_i[x]);
  for (int o = 1; o < kFusedThreads; o <<= 1) {
    const double add = tid >= o ? scan[tid - o] : 0.0;
    __syncthreads();
    scan[tid] += add;
    __syncthreads();
  }
  const double S = scan[kFusedThreads - 1];
  if (argmax_mode) {
    if (tid == 0) {
      x_hat[row] = I;
      if (argmax) argmax[row] = I;
      pmax[row] = (float)(1.0 / S);
      ent[row] = (float)log(S);
    }
    return;
  }
  double A = 0.0;
  int lastpos = -1;
  for (int x = 0; x < kFusedThreads / 32; ++x) { A += red_a[x]; lastpos = max(lastpos, red_l[x]); }
  const Philox4 wd = sampler_words(seed, (uint32_t)i, step, block, (uint32_t)req_ids[b]);
  const double target = (double)unit_uniform(wd.w[0]) * S;
  if (tid == 0) {
    sh_g = 0x7fffffff;
    if (argmax) argmax[row] = I;
    pmax[row] = (float)(1.0 / S);
    ent[row] = (float)(log(S) - A / S);
  }
  __syncthreads();
  const double before = scan[tid] - wt;
  if (before <= target && before + wt > target) {
    double cum = before;
    int gs = -1, glast = -1;
    double p0 = 0.0, p0_last = 0.0;
    for (int g = g0; g < g1; ++g) {
      const VocabStat p = pr[g];
      const double c = (double)p.s * exp((double)p.m - (double)M);
      if (c > 0.0) { glast = g; p0_last = cum; }
      if (cum + c > target) { gs = g; p0 = cum; break; }
      cum += c;
    }
    if (gs < 0) { gs = glast; p0 = p0_last; }   // the thread's sum crossed, the group walk fell short
    sh_g = gs;
    sh_P0 = p0;
  }
  __syncthreads();
  if (sh_g == 0x7fffffff) {
    // no crossing (rounding): the last group with mass, walked to its last positive entry
    if (tid == 0) { sh_g = lastpos; sh_P0 = INFINITY; }
    __syncthreads();
  }
  const int gsel = sh_g;
  // recompute the group's logits: warp w takes rows 4w .. 4w+3 of the group
  const __nv_bfloat16* x = xn + (size_t)row * d;
  for (int u = 0; u < kGroup / (kFusedThreads / 32); ++u) {
    const int v = gsel * kGroup + w * (kGroup / (kFusedThreads / 32)) + u;
    float acc = 0.f;
    if (v < vocab) {
      const __nv_bfloat16* er = emb + (size_t)v * d;
      for (int k = lane * 8; k < d; k += 32 * 8) {
        const uint4 xa = *reinterpret_cast<const uint4*>(x + k);
        const uint4 ea = *reinterpret_cast<const uint4*>(er + k);
        const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
        const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&ea);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 xf = __bfloat1622float2(x2[q]), ef = __bfloat1622float2(e2[q]);
          acc = fmaf(xf.x, ef.x, acc);
          acc = fmaf(xf.y, ef.y, acc);
        }
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) sh_z[w * (kGroup / (kFusedThreads / 32)) + u] = v < vocab ? acc * scale : -INFINITY;
  }
  __syncthreads();
  if (tid == 0) {
    double cum = sh_P0;
    int pick = -1, last = -1;
    for (int j = 0; j < kGroup; ++j) {
      const float e = expf(sh_z[j] - M);
      if (e > 0.f) last = j;
      cum += (double)e;
      if (pick < 0 && cum > target) pick = j;
    }
    if (pick < 0) pick = last >= 0 ? last : 0;
    x_hat[row] = gsel * kGroup + pick;
  }
}

void launch_sampler_fused_rows(const VocabStat* stats, int n_groups, const __nv_bfloat16* xn,
                               const __nv_bfloat16* embed, int d, int rows, int n, int vocab, const int* req_ids,
                               const SamplerArgs& a, int32_t* x_hat, float* pmax, float* ent, cudaStream_t s,
                               int32_t* argmax) {
  if (rows <= 0) return;
  const int argmax_mode = a.temperature == 0.f;
  const float scale = argmax_mode ? a.logit_scale : a.logit_scale / a.temperature;
  launch_k(sampler_pass2_fused, dim3(rows), dim3(kFusedThreads), 0, s, stats, n_groups, xn, embed, d, n, vocab, scale,
           argmax_mode, req_ids, a.seed, a.step, a.block, x_hat, pmax, ent, argmax);
}

// Pass 3: per canvas.  Top-k keep: rank_i = #{j : pmax_j > pmax_i or
// (pmax_j == pmax_i and j < i)}, kept iff rank_i < keep_k.  Entropy budget:
// r_i = #{j : H_j < H_i or (H_j == H_i and j < i)} orders the positions by
// entropy; C_i = sum of H_j over r_j <= r_i (fp64) is the running sum that
// reaches position i, and the positions kept are those ranked before the first
// one whose C exceeds the budget (a running sum of H >= 0 only grows, so that
// is also where it stays above).  Rank 0, where locking starts, is always kept.
// Two-round stop: this round's and the previous round's mean entropies below
// the threshold and every position's arg-max unchanged; no previous round, no
// stop.
__global__ void sampler_finish_kernel(const int32_t* __restrict__ x_hat, const float* __restrict__ pmax,
                                      const float* __restrict__ ent, int n, int vocab, const int* __restrict__ req_ids,
                                      uint64_t seed, uint32_t step, uint32_t block, int keep_k, int keep_mode,
                                      float budget, float stop_thr, int stop_mode,
                                      const int32_t* __restrict__ amax_cur, const int32_t* __restrict__ amax_prev,
                                      const float* __restrict__ mh_prev,
                                      int32_t* __restrict__ canvas, int32_t* __restrict__ keep_out,
                                      float* __restrict__ mean_h, int32_t* __restrict__ stop_out,
                                      int32_t* __restrict__ done, int32_t* __restrict__ out_tokens, int final_step) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float pm[];  // [n] pmax, then [n] entropy for the budget keep
  float* eh = pm + n;
  __shared__ float red[32];
  __shared__ int sh_stop;
  __shared__ int sh_cut;         // budget keep: entropy rank of the first position re-noised
  const int b = blockIdx.x;
  const int req = req_ids[b];
  const int i = threadIdx.x;
  for (int j = i; j < n; j += blockDim.x) {
    pm[j] = pmax[(size_t)b * n + j];
    if (keep_mode == 1) eh[j] = ent[(size_t)b * n + j];
  }
  if (i == 0) sh_cut = n;
  const int was_done = (done != nullptr) ? done[b] : 0;
  __syncthreads();
  int same = 1;
  if (stop_mode == 1) {  // uniform over the block
    int eq = 1;
    if (amax_prev != nullptr && i < n) eq = amax_cur[(size_t)b * n + i] == amax_prev[(size_t)b * n + i];
    same = __syncthreads_and(eq);
  }
  int hrank = 0;
  if (keep_mode == 1 && i < n) {
    const float h = eh[i];
    double run = 0.0;
    for (int j = 0; j < n; ++j) {
      const float q = eh[j];
      const int before = (q < h || (q == h && j < i)) ? 1 : 0;
      hrank += before;
      if (before || j == i) run += (double)q;
    }
    if (run > (double)budget) atomicMin(&sh_cut, hrank);
  }
  float hsum = 0.f;
  if (i < n) hsum = ent[(size_t)b * n + i];
  // deterministic block sum over positions
  hsum = warp_sum(hsum);
  if ((i & 31) == 0) red[i >> 5] = hsum;
  __syncthreads();
  if (i == 0) {
    float t = 0.f;
    for (int x = 0; x < (int)((blockDim.x + 31) >> 5); ++x) t += red[x];
    const float mh = t / (float)n;
    int st;
    if (stop_mode == 1)
      st = (stop_thr >= 0.f && amax_prev != nullptr && mh_prev != nullptr && mh_prev[b] < stop_thr &&
            mh < stop_thr && same) ? 1 : 0;
    else
      st = (stop_thr >= 0.f && mh < stop_thr) ? 1 : 0;
    if (mean_h) mean_h[b] = mh;
    if (stop_out) stop_out[b] = st;
    sh_stop = st;
  }
  __syncthreads();
  if (i < n) {
    int kept;
    if (keep_mode == 1) {
      kept = hrank < max(sh_cut, 1);
    } else {
      const float p = pm[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const float q = pm[j];
        rank += (q > p || (q == p && j < i)) ? 1 : 0;
      }
      kept = rank < keep_k;
    }
    const int32_t xh = x_hat[(size_t)b * n + i];
    const Philox4 w = sampler_words(seed, (uint32_t)i, step, block, (uint32_t)req);
    const int32_t tok = kept ? xh : uniform_token(w.w[1], (uint32_t)vocab);
    canvas[(size_t)b * n + i] = tok;
    if (keep_out) keep_out[(size_t)b * n + i] = kept;
    if (out_tokens != nullptr && !was_done && (sh_stop || final_step)) out_tokens[(size_t)b * n + i] = xh;
  }
  __syncthreads();
  if (i == 0 && done != nullptr && !was_done && (sh_stop || final_step)) done[b] = 1;
}

void launch_sampler_finish(const int32_t* x_hat, const float* pmax, const float* ent, int B, int n, int vocab,
                           const int* req_ids, const SamplerArgs& a, int32_t* canvas, int32_t* keep, float* mean_h,
                           int32_t* stop, int32_t* done, int32_t* out_tokens, int final_step, cudaStream_t s,
                           const int32_t* argmax) {
  if (B <= 0) return;
  const int threads = ((n + 31) / 32) * 32;
  const int keep_mode = a.keep_mode == 1 ? 1 : 0;
  const int stop_mode = (a.stop_mode == 1 && argmax != nullptr) ? 1 : 0;
  const size_t smem = (size_t)n * sizeof(float) * (keep_mode ? 2 : 1);
  launch_k(sampler_finish_kernel, dim3(B), dim3(threads), smem, s, x_hat, pmax, ent, n, vocab, req_ids, a.seed, a.step,
                                                              a.block, a.keep_k, keep_mode, a.entropy_budget,
                                                              a.stop_threshold, stop_mode, argmax, a.prev_argmax,
                                                              a.prev_mean_h, canvas, keep,
                                                              mean_h, stop, done, out_tokens, final_step);
}

// ------------------------------------------------------------ self test
__global__ void philox_selftest_kernel(const uint32_t* ctr, const uint32_t* key, uint32_t* out,
                                       uint32_t* out_curand, int n) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const Philox4 o = philox4x32_10(ctr[4 * t], ctr[4 * t + 1], ctr[4 * t + 2], ctr[4 * t + 3], key[2 * t],
                                  key[2 * t + 1]);
  for (int j = 0; j < 4; ++j) out[4 * t + j] = o.w[j];
  if (out_curand) {
    const uint4 c = make_uint4(ctr[4 * t], ctr[4 * t + 1], ctr[4 * t + 2], ctr[4 * t + 3]);
    const uint2 k = make_uint2(key[2 * t], key[2 * t + 1]);
    const uint4 r = curand_Philox4x32_10(c, k);
    out_curand[4 * t] = r.x;
    out_curand[4 * t + 1] = r.y;
    out_curand[4 * t + 2] = r.z;
    out_curand[4 * t + 3] = r.w;
  }
}

void launch_philox_selftest(const uint32_t* ctr, const uint32_t* key, uint32_t* out, uint32_t* out_curand, int n,
                            cudaStream_t s) {
  if (n <= 0) return;
  launch_k(philox_selftest_kernel, dim3((n + 127) / 128), dim3(128), 0, s, ctr, key, out, out_curand, n);
}

}  // namespace dg
