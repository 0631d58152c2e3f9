// Single-token attention for AR-mode decode ([P1 七]: the diffusion model's
// weights load unchanged as an autoregressive model; [P1 五] compares canvas
// attention with this single-token attention).  One new query per request and
// query head attends to the whole cache [0, P] (the new token's own K/V at
// position P included): there is nothing to mask and no query tile, so the
// work is one pass over the cache, bound by HBM.
//
// One CTA per (key split, KV head, request) serves all G = Hq/Hkv query heads
// of that KV head (GQA sharing: each K/V byte is read once per request).  Keys
// are taken in chunks of 64:
//   - scores: each warp owns 8 keys; a lane holds 8 of the 256 head
//     dimensions and loads its 16 bytes of each key row (a warp reads whole
//     512-byte rows); the warp sums the G dot products with shuffles;
//   - online softmax: warp g updates head g's running max and sum (log2 units);
//   - P.V: thread d owns output dimension d and reads the chunk's 64
//     consecutive keys of its row of the transposed V cache (128 bytes) once
//     for all G heads.
// The split partials (unnormalised O, max, sum) go to the workspace and the
// combine kernel of the canvas attention's KV splits.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

constexpr int kDecHd = 256;
constexpr int kDecThreads = 256;
constexpr int kDecChunk = 64;

struct AttnDecodeParams {
  AttnArgs a;
  int n_split;
  int per;                   // keys per split, a multiple of kDecChunk
  float scale_log2;          // log2(e) / sqrt(hd)
  const __nv_bfloat16* q;    // [B][Hq][1][hd]
  const __nv_bfloat16* kc;   // [slots][Hkv][max_ctx][hd]
  const __nv_bfloat16* vt;   // [slots][Hkv][hd][max_ctx]
  float* part_o;             // [n_split][B * Hq][hd]
  float* part_ml;            // [n_split][B * Hq][2]
};

template <int G>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(const AttnDecodeParams P) {
  __shared__ float sq[G][kDecHd];
  __shared__ float ss[G][kDecChunk];
  __shared__ float s_m[G], s_l[G], s_alpha[G];
  const AttnArgs& a = P.a;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slot = a.bi.slot[b];
  const int nkeys = a.bi.len[b] + 1;                        // the cache and the new token
  const int j0 = min(nkeys, split * P.per), j1 = min(nkeys, j0 + P.per);
  const size_t rows = (size_t)a.B * a.hq;
  const size_t row0 = (size_t)b * a.hq + (size_t)kvh * G;  // first query head of this KV head
  pdl_wait();
  pdl_trigger();
  for (int i = tid; i < G * kDecHd; i += kDecThreads) sq[i / kDecHd][i % kDecHd] = __bfloat162float(P.q[row0 * kDecHd + i]);
  if (tid < G) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  __syncthreads();
  float qr[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) qr[g][e] = sq[g][lane * 8 + e];
  const __nv_bfloat16* kbase = P.kc + ((size_t)slot * a.hkv + kvh) * a.max_ctx * kDecHd;
  const __nv_bfloat16* vrow = P.vt + (((size_t)slot * a.hkv + kvh) * kDecHd + tid) * a.max_ctx;
  float o[G];
#pragma unroll
  for (int g = 0; g < G; ++g) o[g] = 0.f;

  for (int c0 = j0; c0 < j1; c0 += kDecChunk) {
    const int nc = min(kDecChunk, j1 - c0);
    uint4 kv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int jj = warp * 8 + u;
      kv[u] = jj < nc ? *reinterpret_cast<const uint4*>(kbase + (size_t)(c0 + jj) * kDecHd + lane * 8)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int jj = warp * 8 + u;
      const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv[u]);
      float kf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(k2[e]);
        kf[2 * e] = f.x;
        kf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(qr[g][e], kf[e], s);
        s = warp_sum(s);
        if (lane == 0) ss[g][jj] = jj < nc ? s * P.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();
    if (warp < G) {
      const int g = warp;
      const float x0 = ss[g][lane], x1 = ss[g][lane + 32];
      const float m_old = s_m[g];
      const float mn = fmaxf(m_old, warp_max(fmaxf(x0, x1)));   // finite: the chunk has a key
      const float p0 = exp2f(x0 - mn), p1 = exp2f(x1 - mn);
      ss[g][lane] = p0;
      ss[g][lane + 32] = p1;
      const float cs = warp_sum(p0 + p1);
      if (lane == 0) {
        const float al = exp2f(m_old - mn);                      // 0 at the first chunk
        s_alpha[g] = al;
        s_l[g] = s_l[g] * al + cs;
        s_m[g] = mn;
      }
    }
    __syncthreads();
    const __nv_bfloat16* vp = vrow + c0;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    for (int j = 0; j < nc; j += 8) {
      __nv_bfloat16 vv[8];
      if (j + 8 <= nc) {
        *reinterpret_cast<uint4*>(vv) = *reinterpret_cast<const uint4*>(vp + j);   // c0, j multiples of 8
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) vv[e] = j + e < nc ? vp[j + e] : __float2bfloat16_rn(0.f);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = __bfloat162float(vv[e]);
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = fmaf(ss[g][j + e], v, acc[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) o[g] = o[g] * s_alpha[g] + acc[g];
    __syncthreads();   // ss is rewritten by the next chunk
  }
  // an empty split (j0 == j1) leaves m = -inf, l = 0, o = 0: the combine skips it
#pragma unroll
  for (int g = 0; g < G; ++g) P.part_o[((size_t)split * rows + row0 + g) * kDecHd + tid] = o[g];
  if (tid < G) {
    P.part_ml[2 * ((size_t)split * rows + row0 + tid)] = s_m[tid];
    P.part_ml[2 * ((size_t)split * rows + row0 + tid) + 1] = s_l[tid];
  }
}

int attn_decode_splits(int B, int hkv, int max_keys, int num_sms, size_t part_rows_cap, int hq) {
  const int chunks = (max_keys + kDecChunk - 1) / kDecChunk;
  int n = (2 * num_sms + B * hkv - 1) / (B * hkv);
  n = std::max(1, std::min(n, std::min(64, chunks)));
  while (n > 1 && (size_t)n * B * hq > part_rows_cap) --n;
  return n;
}

int launch_attn_decode(const __nv_bfloat16* q, const __nv_bfloat16* kc, const __nv_bfloat16* vt,
                       __nv_bfloat16* out, const AttnArgs& a, float* part_o, float* part_ml, size_t part_rows_cap,
                       int num_sms, cudaStream_t s) {
  if (a.B <= 0) return 0;
  if (a.nq != 1 || a.hd != kDecHd) return -1;
  const int G = a.hq / a.hkv;
  int max_keys = 0;
  for (int b = 0; b < a.B; ++b) max_keys = std::max(max_keys, a.bi.len[b] + 1);
  AttnDecodeParams P;
  P.a = a;
  P.n_split = attn_decode_splits(a.B, a.hkv, max_keys, num_sms, part_rows_cap, a.hq);
  const int chunks = (max_keys + kDecChunk - 1) / kDecChunk;
  P.per = ((chunks + P.n_split - 1) / P.n_split) * kDecChunk;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)a.hd);
  P.q = q;
  P.kc = kc;
  P.vt = vt;
  P.part_o = part_o;
  P.part_ml = part_ml;
  const dim3 grid(P.n_split, a.hkv, a.B);
  switch (G) {
    case 1: launch_k(attn_decode_kernel<1>, grid, dim3(kDecThreads), 0, s, P); break;
    case 2: launch_k(attn_decode_kernel<2>, grid, dim3(kDecThreads), 0, s, P); break;
    case 4: launch_k(attn_decode_kernel<4>, grid, dim3(kDecThreads), 0, s, P); break;
    case 8: launch_k(attn_decode_kernel<8>, grid, dim3(kDecThreads), 0, s, P); break;
    default: return -1;
  }
  launch_attn_combine(part_o, part_ml, out, P.n_split, a.B, a.hq, 1, s);
  return 0;
}

}  // namespace dg
