// Small memory-bound kernels of the step: embedding + self-conditioning
// gather, RMSNorm, the MoE combine (fused with the next RMSNorm), the RoPE
// split of the fused QKV output into Q / K-cache / transposed V-cache, the
// row gather into expert order, canvas initialisation and the cache writer.
#include <cuda_bf16.h>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

// ------------------------------------------------------------------ embed
// [P1 二] self-conditioning: the previous step's predictions are embedded and
// later projected by W_sc; here we gather both embedding rows.
// A token outside [0, vocab) is replaced by 0 and recorded in *err (it is
// never used as an address).
__device__ __forceinline__ int checked_token(int32_t x, int vocab, int* err) {
  if (x < 0 || x >= vocab) {
    if (err) atomicCAS(err, 0, kErrBadToken);
    return 0;
  }
  return x;
}

template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tok, const int32_t* __restrict__ prev,
                             const T* __restrict__ embed, float* __restrict__ h, T* __restrict__ eprev, int d,
                             int vocab, int* err) {
  const int t = blockIdx.x;
  const T* e = embed + (size_t)checked_token(tok[t], vocab, err) * d;
  float* ho = h + (size_t)t * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) ho[j] = to_f32(e[j]);
  if (prev != nullptr) {
    const T* ep = embed + (size_t)checked_token(prev[t], vocab, err) * d;
    T* o = eprev + (size_t)t * d;
    for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = ep[j];
  }
}

template <typename T>
void launch_embed(const int32_t* tok, const int32_t* prev, const T* embed, float* h, T* eprev, int n_tok, int d,
                  int vocab, int* err, cudaStream_t s) {
  if (n_tok <= 0) return;
  embed_kernel<T><<<n_tok, 256, 0, s>>>(tok, prev, embed, h, eprev, d, vocab, err);
}

// ------------------------------------------------------------ block reduce
// Deterministic block sum: fixed tree over warps.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  float r = 0.f;
  if (w == 0) {
    r = (l < nw) ? red[l] : 0.f;
    r = warp_sum(r);
    if (l == 0) red[0] = r;
  }
  __syncthreads();
  r = red[0];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------- RMSNorm
// Rows are processed as float4 when d % 4 == 0 (16-byte loads), else as floats.
template <typename T>
__device__ __forceinline__ void store4(T* o, int j4, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* o, int j4, float4 v) {
  reinterpret_cast<float4*>(o)[j4] = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* o, int j4, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  reinterpret_cast<uint2*>(o)[j4] = u;
}

template <typename T>
__global__ void rmsnorm_kernel(const float* __restrict__ h, const float* __restrict__ w, T* __restrict__ xn,
                               int d, float eps) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* x = h + (size_t)t * d;
  T* o = xn + (size_t)t * d;
  float ss = 0.f;
  if ((d & 3) == 0) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    for (int j = threadIdx.x; j < d / 4; j += blockDim.x) {
      const float4 v = x4[j];
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
    const float4* w4 = reinterpret_cast<const float4*>(w);
    for (int j = threadIdx.x; j < d / 4; j += blockDim.x) {
      const float4 v = x4[j], g = w4[j];
      store4<T>(o, j, make_float4(v.x * r * g.x, v.y * r * g.y, v.z * r * g.z, v.w * r * g.w));
    }
    return;
  }
  for (int j = threadIdx.x; j < d; j += blockDim.x) ss += x[j] * x[j];
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
  for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = from_f32<T>(x[j] * r * w[j]);
}

template <typename T>
void launch_rmsnorm(const float* h, const float* w, T* xn, int n_tok, int d, float eps, cudaStream_t s) {
  if (n_tok <= 0) return;
  rmsnorm_kernel<T><<<n_tok, 256, 0, s>>>(h, w, xn, d, eps);
}

// ---------------------------------------------------------------- combine
// h[t] += sum over the k slots, in slot order, of w[t,s] * y[t*k+s]; then the
// optional RMSNorm of the new residual into xn.  Each element is owned by one
// thread and summed in slot order: no atomics, bitwise reproducible.  The
// float4 path issues the k slot loads of a column group together.
template <typename T>
__global__ void combine_kernel(float* __restrict__ h, const float* __restrict__ y, const float* __restrict__ wts,
                               int k, const float* __restrict__ norm_w, T* __restrict__ xn, int d, float eps) {
  __shared__ float red[32];
  __shared__ float ws[16];
  const int t = blockIdx.x;
  if (threadIdx.x < k) ws[threadIdx.x] = wts[(size_t)t * k + threadIdx.x];
  __syncthreads();
  float* hr = h + (size_t)t * d;
  const float* yr = y + (size_t)t * k * d;
  float ss = 0.f;
  if ((d & 3) == 0) {
    const int d4 = d / 4;
    float4* h4 = reinterpret_cast<float4*>(hr);
    const float4* y4 = reinterpret_cast<const float4*>(yr);
    for (int j = threadIdx.x; j < d4; j += blockDim.x) {
      float4 yv[16];
#pragma unroll
      for (int s = 0; s < 16; ++s)
        if (s < k) yv[s] = y4[(size_t)s * d4 + j];
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 16; ++s)
        if (s < k) {
          acc.x += ws[s] * yv[s].x;
          acc.y += ws[s] * yv[s].y;
          acc.z += ws[s] * yv[s].z;
          acc.w += ws[s] * yv[s].w;
        }
      float4 v = h4[j];
      v.x += acc.x; v.y += acc.y; v.z += acc.z; v.w += acc.w;
      h4[j] = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    if (norm_w == nullptr) return;
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
    const float4* w4 = reinterpret_cast<const float4*>(norm_w);
    T* o = xn + (size_t)t * d;
    for (int j = threadIdx.x; j < d4; j += blockDim.x) {
      const float4 v = h4[j], g = w4[j];
      store4<T>(o, j, make_float4(v.x * r * g.x, v.y * r * g.y, v.z * r * g.z, v.w * r * g.w));
    }
    return;
  }
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < k; ++s) acc += ws[s] * yr[(size_t)s * d + j];
    const float v = hr[j] + acc;
    hr[j] = v;
    ss += v * v;
  }
  if (norm_w == nullptr) return;
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
  T* o = xn + (size_t)t * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = from_f32<T>(hr[j] * r * norm_w[j]);
}

template <typename T>
void launch_combine(float* h, const float* y, const float* wts, int k, const float* norm_w, T* xn, int n_tok,
                    int d, float eps, cudaStream_t s) {
  if (n_tok <= 0) return;
  combine_kernel<T><<<n_tok, 256, 0, s>>>(h, y, wts, k, norm_w, xn, d, eps);
}

// ------------------------------------------------------------ RoPE scatter
// Rotate-half RoPE at absolute position len[b] + i ([P1 二]: the canvas
// continues the prompt's positions).  rope_cs[pos][j] = (cos, sin) of
// pos * base^(-2j/hd), tabulated on the host in double precision.
template <typename T>
__global__ void rope_scatter_kernel(const float* __restrict__ qkv, T* __restrict__ q, T* __restrict__ kc,
                                    T* __restrict__ vt, const float2* __restrict__ rope_cs, BatchInfo bi, int nq,
                                    int hq, int hkv, int hd, int max_ctx) {
  const int t = blockIdx.x;            // token row b*nq + i
  const int head = blockIdx.y;         // 0..hq+2hkv-1
  const int b = t / nq, i = t - b * nq;
  const int pos = bi.len[b] + i;
  const int slot = bi.slot[b];
  const int half = hd >> 1;
  const int ncol = (hq + 2 * hkv) * hd;
  const float* src = qkv + (size_t)t * ncol + (size_t)head * hd;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const float x1 = src[j], x2 = src[j + half];
    if (head < hq + hkv) {
      const float2 cs = rope_cs[(size_t)pos * half + j];
      const float r1 = x1 * cs.x - x2 * cs.y;
      const float r2 = x2 * cs.x + x1 * cs.y;
      T* dst;
      if (head < hq) {
        dst = q + (((size_t)b * hq + head) * nq + i) * hd;
      } else {
        const int g = head - hq;
        dst = kc + (((size_t)slot * hkv + g) * max_ctx + pos) * hd;
      }
      dst[j] = from_f32<T>(r1);
      dst[j + half] = from_f32<T>(r2);
    } else {
      const int g = head - hq - hkv;
      T* dst = vt + ((size_t)slot * hkv + g) * hd * (size_t)max_ctx + pos;
      dst[(size_t)j * max_ctx] = from_f32<T>(x1);
      dst[(size_t)(j + half) * max_ctx] = from_f32<T>(x2);
    }
  }
}

template <typename T>
void launch_rope_scatter(const float* qkv, T* q, T* kc, T* vt, const float* rope_cs, const BatchInfo& bi,
                         int nq, int hq, int hkv, int hd, int max_ctx, cudaStream_t s) {
  const int n_tok = bi.B * nq;
  if (n_tok <= 0) return;
  dim3 grid(n_tok, hq + 2 * hkv);
  rope_scatter_kernel<T><<<grid, 128, 0, s>>>(qkv, q, kc, vt, reinterpret_cast<const float2*>(rope_cs), bi,
                                              nq, hq, hkv, hd, max_ctx);
}

// ------------------------------------------------------------ gather rows
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ xn, const int32_t* __restrict__ perm, T* __restrict__ xp,
                                   int k, int d) {
  const int p = blockIdx.x;
  const int src = perm[p] / k;
  // 16-byte vectors when the row is 16-byte aligned (d * sizeof(T) % 16 == 0)
  if ((d * sizeof(T)) % 16 == 0) {
    const int nv = d * (int)sizeof(T) / 16;
    const uint4* s4 = reinterpret_cast<const uint4*>(xn + (size_t)src * d);
    uint4* d4 = reinterpret_cast<uint4*>(xp + (size_t)p * d);
    for (int j = threadIdx.x; j < nv; j += blockDim.x) d4[j] = s4[j];
  } else {
    for (int j = threadIdx.x; j < d; j += blockDim.x) xp[(size_t)p * d + j] = xn[(size_t)src * d + j];
  }
}

template <typename T>
void launch_gather_rows(const T* xn, const int32_t* perm, T* xp, int n_rows, int k, int d, cudaStream_t s) {
  if (n_rows <= 0) return;
  gather_rows_kernel<T><<<n_rows, 128, 0, s>>>(xn, perm, xp, k, d);
}

// ------------------------------------------------------------ init canvas
// [P1 一], [P2 运作机制]: the canvas starts as uniform-random vocabulary tokens.
__global__ void init_canvas_kernel(int32_t* canvas, BatchInfo bi, const int* req_ids, int n, int vocab,
                                   uint64_t seed, uint32_t block) {
  const int b = blockIdx.x;
  const int req = bi.slot[b];
  (void)req_ids;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const Philox4 w = sampler_words(seed, (uint32_t)i, 0u, block, (uint32_t)req);
    canvas[(size_t)b * n + i] = uniform_token(w.w[1], (uint32_t)vocab);
  }
}

void launch_init_canvas(int32_t* canvas, const BatchInfo& bi, const int* req_ids, int n, int vocab, uint64_t seed,
                        uint32_t block, cudaStream_t s) {
  if (bi.B <= 0) return;
  init_canvas_kernel<<<bi.B, 256, 0, s>>>(canvas, bi, req_ids, n, vocab, seed, block);
}

// ----------------------------------------------------------------- set_kv
template <typename T>
__global__ void set_kv_kernel(const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ kc,
                              T* __restrict__ vt, int n, int hd, int max_ctx) {
  const int g = blockIdx.y;
  const int p = blockIdx.x;
  for (int j = threadIdx.x; j < hd; j += blockDim.x) {
    kc[((size_t)g * max_ctx + p) * hd + j] = k[((size_t)g * n + p) * hd + j];
    vt[((size_t)g * hd + j) * max_ctx + p] = v[((size_t)g * n + p) * hd + j];
  }
}

template <typename T>
void launch_set_kv(const T* k, const T* v, T* kc, T* vt, int hkv, int n, int hd, int max_ctx, cudaStream_t s) {
  if (n <= 0) return;
  set_kv_kernel<T><<<dim3(n, hkv), 128, 0, s>>>(k, v, kc, vt, n, hd, max_ctx);
}

// ------------------------------------------------------------ instantiation
#define DG_INST(T)                                                                                          \
  template void launch_embed<T>(const int32_t*, const int32_t*, const T*, float*, T*, int, int, int, int*,    \
                                cudaStream_t);                                                             \
  template void launch_rmsnorm<T>(const float*, const float*, T*, int, int, float, cudaStream_t);            \
  template void launch_combine<T>(float*, const float*, const float*, int, const float*, T*, int, int, float, \
                                  cudaStream_t);                                                             \
  template void launch_rope_scatter<T>(const float*, T*, T*, T*, const float*, const BatchInfo&, int, int, int, \
                                       int, int, cudaStream_t);                                              \
  template void launch_gather_rows<T>(const T*, const int32_t*, T*, int, int, int, cudaStream_t);            \
  template void launch_set_kv<T>(const T*, const T*, T*, T*, int, int, int, int, cudaStream_t);
DG_INST(float)
DG_INST(__nv_bfloat16)
#undef DG_INST

}  // namespace dg
