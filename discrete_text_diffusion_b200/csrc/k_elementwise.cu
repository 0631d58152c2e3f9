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
  pdl_wait();
  pdl_trigger();
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
  launch_k(embed_kernel<T>, dim3(n_tok), dim3(256), 0, s, tok, prev, embed, h, eprev, d, vocab, err);
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

// Four consecutive elements j4*4 .. j4*4+3 of a row as floats (16- or 8-byte load).
template <typename T>
__device__ __forceinline__ float4 load4(const T* p, size_t j4);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p, size_t j4) {
  return reinterpret_cast<const float4*>(p)[j4];
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p, size_t j4) {
  const uint2 u = reinterpret_cast<const uint2*>(p)[j4];
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

template <typename T>
__global__ void rmsnorm_kernel(const float* __restrict__ h, const float* __restrict__ w, T* __restrict__ xn,
                               int d, float eps) {
  pdl_wait();
  pdl_trigger();
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

// Register-resident rows: thread x owns float4 columns x, x + blockDim, ...
// (VPT of them), so a row is read from memory once and normalised from
// registers.  One CTA per row, blockDim = ceil(d / 4 / VPT) rounded to a warp.
constexpr int kRowThreadsMax = 1024;

__host__ __device__ constexpr int row_threads(int d4, int vpt) { return ((d4 + vpt - 1) / vpt + 31) / 32 * 32; }

inline int row_vpt(int d) {
  if (d % 4 != 0) return 0;
  const int d4 = d / 4;
  for (int v = 1; v <= 8; v *= 2)
    if (row_threads(d4, v) <= kRowThreadsMax) return v;
  return 0;
}

template <typename T, int VPT>
__global__ void __launch_bounds__(kRowThreadsMax) rmsnorm_reg_kernel(const float* __restrict__ h,
                                                                     const float* __restrict__ w,
                                                                     T* __restrict__ xn, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int t = blockIdx.x, d4 = d >> 2;
  const float4* x4 = reinterpret_cast<const float4*>(h + (size_t)t * d);
  float4 v[VPT];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int j = threadIdx.x + u * blockDim.x;
    v[u] = j < d4 ? x4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
  }
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
  const float4* w4 = reinterpret_cast<const float4*>(w);
  T* o = xn + (size_t)t * d;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int j = threadIdx.x + u * blockDim.x;
    if (j < d4) {
      const float4 g = w4[j];
      store4<T>(o, j, make_float4(v[u].x * r * g.x, v[u].y * r * g.y, v[u].z * r * g.z, v[u].w * r * g.w));
    }
  }
}

template <typename T>
void launch_rmsnorm(const float* h, const float* w, T* xn, int n_tok, int d, float eps, cudaStream_t s) {
  if (n_tok <= 0) return;
  const int vpt = row_vpt(d);
  const int thr = vpt ? row_threads(d / 4, vpt) : 256;
  switch (vpt) {
    case 1: launch_k(rmsnorm_reg_kernel<T, 1>, dim3(n_tok), dim3(thr), 0, s, h, w, xn, d, eps); break;
    case 2: launch_k(rmsnorm_reg_kernel<T, 2>, dim3(n_tok), dim3(thr), 0, s, h, w, xn, d, eps); break;
    case 4: launch_k(rmsnorm_reg_kernel<T, 4>, dim3(n_tok), dim3(thr), 0, s, h, w, xn, d, eps); break;
    case 8: launch_k(rmsnorm_reg_kernel<T, 8>, dim3(n_tok), dim3(thr), 0, s, h, w, xn, d, eps); break;
    default: launch_k(rmsnorm_kernel<T>, dim3(n_tok), dim3(256), 0, s, h, w, xn, d, eps);
  }
}

// Residual add of split-K partial sums, then RMSNorm.  Each thread owns VPT
// float4 columns; the slices are added in slice order.  VPT 0 is the generic
// form: any d, columns strided over the block, the row re-read for the norm.
template <typename T, int VPT>
__global__ void __launch_bounds__(kRowThreadsMax) add_rmsnorm_kernel(float* __restrict__ h,
                                                                     const float* __restrict__ part, int nsplit,
                                                                     size_t split_stride,
                                                                     const float* __restrict__ w,
                                                                     T* __restrict__ xn, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int t = blockIdx.x;
  float* hr = h + (size_t)t * d;
  const float* pr = part + (size_t)t * d;
  T* o = xn + (size_t)t * d;
  float ss = 0.f;
  if constexpr (VPT == 0) {
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      float a = 0.f;
      for (int sp = 0; sp < nsplit; ++sp) a += pr[(size_t)sp * split_stride + j];
      const float x = hr[j] + a;
      hr[j] = x;
      ss += x * x;
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
    for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = from_f32<T>(hr[j] * r * w[j]);
  } else {
    const int d4 = d >> 2;
    float4* h4 = reinterpret_cast<float4*>(hr);
    const float4* p4 = reinterpret_cast<const float4*>(pr);
    const size_t s4 = split_stride / 4;
    float4 v[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int j = threadIdx.x + u * blockDim.x;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < d4) {
        float4 a = p4[j];
        for (int sp0 = 1; sp0 < nsplit; sp0 += 4) {
          float4 b[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (sp0 + q < nsplit) b[q] = p4[(size_t)(sp0 + q) * s4 + j];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (sp0 + q < nsplit) { a.x += b[q].x; a.y += b[q].y; a.z += b[q].z; a.w += b[q].w; }
        }
        float4 x = h4[j];
        x.x += a.x; x.y += a.y; x.z += a.z; x.w += a.w;
        h4[j] = x;
        v[u] = x;
        ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      }
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)d + eps);
    const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int j = threadIdx.x + u * blockDim.x;
      if (j < d4) {
        const float4 g = w4[j];
        store4<T>(o, j, make_float4(v[u].x * r * g.x, v[u].y * r * g.y, v[u].z * r * g.z, v[u].w * r * g.w));
      }
    }
  }
}

template <typename T>
void launch_add_rmsnorm(float* h, const float* part, int nsplit, size_t split_stride, const float* w, T* xn,
                        int n_tok, int d, float eps, cudaStream_t s) {
  if (n_tok <= 0) return;
  const int vpt = (split_stride % 4 == 0) ? row_vpt(d) : 0;
  const int thr = vpt ? row_threads(d / 4, vpt) : 256;
  switch (vpt) {
    case 1: launch_k(add_rmsnorm_kernel<T, 1>, dim3(n_tok), dim3(thr), 0, s, h, part, nsplit, split_stride, w, xn, d, eps); break;
    case 2: launch_k(add_rmsnorm_kernel<T, 2>, dim3(n_tok), dim3(thr), 0, s, h, part, nsplit, split_stride, w, xn, d, eps); break;
    case 4: launch_k(add_rmsnorm_kernel<T, 4>, dim3(n_tok), dim3(thr), 0, s, h, part, nsplit, split_stride, w, xn, d, eps); break;
    case 8: launch_k(add_rmsnorm_kernel<T, 8>, dim3(n_tok), dim3(thr), 0, s, h, part, nsplit, split_stride, w, xn, d, eps); break;
    default: launch_k(add_rmsnorm_kernel<T, 0>, dim3(n_tok), dim3(thr), 0, s, h, part, nsplit, split_stride, w, xn, d, eps);
  }
}

// ---------------------------------------------------------------- combine
// h[t] += sum over the k slots, in slot order, of w[t,s] * y[t*k+s]; then the
// optional RMSNorm of the new residual into xn.  Each element is owned by one
// thread and summed in slot order: no atomics, bitwise reproducible.  The
// float4 path issues the k slot loads of a column group together.
template <typename T>
__global__ void combine_kernel(float* __restrict__ h, const T* __restrict__ y, const float* __restrict__ wts,
                               int k, const float* __restrict__ norm_w, T* __restrict__ xn, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  __shared__ float ws[16];
  const int t = blockIdx.x;
  if (threadIdx.x < k) ws[threadIdx.x] = wts[(size_t)t * k + threadIdx.x];
  __syncthreads();
  float* hr = h + (size_t)t * d;
  const T* yr = y + (size_t)t * k * d;
  float ss = 0.f;
  if ((d & 3) == 0) {
    const int d4 = d / 4;
    float4* h4 = reinterpret_cast<float4*>(hr);

    for (int j = threadIdx.x; j < d4; j += blockDim.x) {
      float4 yv[16];
#pragma unroll
      for (int s = 0; s < 16; ++s)
        if (s < k) yv[s] = load4<T>(yr, (size_t)s * d4 + j);
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
    for (int s = 0; s < k; ++s) acc += ws[s] * to_f32(yr[(size_t)s * d + j]);
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

// Register-resident combine: as combine_kernel, each thread owning VPT float4
// columns; the slot loads of a column are issued four at a time and summed
// in slot order.
template <typename T, int VPT>
__global__ void __launch_bounds__(kRowThreadsMax) combine_reg_kernel(float* __restrict__ h,
                                                                     const T* __restrict__ y,
                                                                     const float* __restrict__ wts, int k,
                                                                     const float* __restrict__ norm_w,
                                                                     T* __restrict__ xn, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  __shared__ float ws[16];
  const int t = blockIdx.x, d4 = d >> 2;
  if (threadIdx.x < k) ws[threadIdx.x] = wts[(size_t)t * k + threadIdx.x];
  __syncthreads();
  float4* h4 = reinterpret_cast<float4*>(h + (size_t)t * d);
  const T* yt = y + (size_t)t * k * d;
  float4 v[VPT];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int j = threadIdx.x + u * blockDim.x;
    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < d4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < k; s0 += 4) {
        float4 yv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (s0 + q < k) yv[q] = load4<T>(yt, (size_t)(s0 + q) * d4 + j);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (s0 + q < k) {
            const float c = ws[s0 + q];
            acc.x += c * yv[q].x;
            acc.y += c * yv[q].y;
            acc.z += c * yv[q].z;
            acc.w += c * yv[q].w;
          }
      }
      float4 x = h4[j];
      x.x += acc.x; x.y += acc.y; x.z += acc.z; x.w += acc.w;
      h4[j] = x;
      v[u] = x;
      ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
    }
  }
  if (norm_w == nullptr) return;
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / (float)d + eps);
  const float4* w4 = reinterpret_cast<const float4*>(norm_w);
  T* o = xn + (size_t)t * d;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int j = threadIdx.x + u * blockDim.x;
    if (j < d4) {
      const float4 g = w4[j];
      store4<T>(o, j, make_float4(v[u].x * r * g.x, v[u].y * r * g.y, v[u].z * r * g.z, v[u].w * r * g.w));
    }
  }
}

template <typename T>
void launch_combine(float* h, const T* y, const float* wts, int k, const float* norm_w, T* xn, int n_tok,
                    int d, float eps, cudaStream_t s) {
  if (n_tok <= 0) return;
  const int vpt = k <= 16 ? row_vpt(d) : 0;
  const int thr = vpt ? row_threads(d / 4, vpt) : 256;
  switch (vpt) {
    case 1: launch_k(combine_reg_kernel<T, 1>, dim3(n_tok), dim3(thr), 0, s, h, y, wts, k, norm_w, xn, d, eps); break;
    case 2: launch_k(combine_reg_kernel<T, 2>, dim3(n_tok), dim3(thr), 0, s, h, y, wts, k, norm_w, xn, d, eps); break;
    case 4: launch_k(combine_reg_kernel<T, 4>, dim3(n_tok), dim3(thr), 0, s, h, y, wts, k, norm_w, xn, d, eps); break;
    case 8: launch_k(combine_reg_kernel<T, 8>, dim3(n_tok), dim3(thr), 0, s, h, y, wts, k, norm_w, xn, d, eps); break;
    default: launch_k(combine_kernel<T>, dim3(n_tok), dim3(256), 0, s, h, y, wts, k, norm_w, xn, d, eps);
  }
}

// ------------------------------------------------------------ RoPE scatter
// Rotate-half RoPE at absolute position len[b] + i ([P1 二]: the canvas
// continues the prompt's positions).  rope_cs[pos][j] = (cos, sin) of
// pos * base^(-2j/hd), tabulated on the host in double precision.
template <typename T>
__global__ void rope_scatter_kernel(const float* __restrict__ qkv, int nsplit, size_t split_stride,
                                    T* __restrict__ q, T* __restrict__ kc,
                                    T* __restrict__ vt, const float2* __restrict__ rope_cs, BatchInfo bi, int nq,
                                    int hq, int hkv, int hd, int max_ctx) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;            // token row b*nq + i
  const int head = blockIdx.y;         // 0..hq+2hkv-1
  const int b = t / nq, i = t - b * nq;
  const int pos = bi.len[b] + i;
  const int slot = bi.slot[b];
  const int half = hd >> 1;
  const int ncol = (hq + 2 * hkv) * hd;
  const float* src = qkv + (size_t)t * ncol + (size_t)head * hd;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    float x1 = src[j], x2 = src[j + half];
    for (int sp = 1; sp < nsplit; ++sp) {
      x1 += src[(size_t)sp * split_stride + j];
      x2 += src[(size_t)sp * split_stride + j + half];
    }
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

// Tiled form: one CTA per (32 token rows, head).  Q and K rows are rotated
// four pairs per thread with 16-byte loads.  V rows are staged in shared
// memory and written transposed, one head dimension per warp instruction with
// lane = token, so consecutive lanes store consecutive cache positions.
constexpr int kRopeTok = 32;

// NS = 1 or 2: exactly NS split-K slices and hd <= 256, so a thread's items
// (at most 4 rotated groups, or 8 V vectors) are all loaded before any is
// used: one memory latency per CTA.  NS = 0: any slice count, item by item.
template <typename T, int NS>
__global__ void __launch_bounds__(256) rope_scatter_tiled_kernel(const float* __restrict__ qkv, int nsplit,
                                                                 size_t split_stride, T* __restrict__ q,
                                                                 T* __restrict__ kc, T* __restrict__ vt,
                                                                 const float2* __restrict__ rope_cs, BatchInfo bi,
                                                                 int nq, int n_tok, int hq, int hkv, int hd,
                                                                 int max_ctx) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char rope_smem[];
  const int t0 = blockIdx.x * kRopeTok;
  const int head = blockIdx.y;
  const int half = hd >> 1, g4 = half >> 2;
  const size_t ncol = (size_t)(hq + 2 * hkv) * hd;
  const int ntk = min(kRopeTok, n_tok - t0);
  if constexpr (NS > 0) {
    if (head < hq + hkv) {
      constexpr int kIt = 4;   // kRopeTok * 256 / 8 groups over 256 threads
      float4 x1[kIt], x2[kIt], a1[kIt], a2[kIt], ca[kIt], cb[kIt];
#pragma unroll
      for (int it = 0; it < kIt; ++it) {
        const int idx = threadIdx.x + it * blockDim.x;
        if (idx < ntk * g4) {
          const int tt = idx / g4, j = (idx - tt * g4) * 4;
          const int t = t0 + tt;
          const int b = t / nq, pos = bi.len[b] + (t - b * nq);
          const float* src = qkv + (size_t)t * ncol + (size_t)head * hd;
          x1[it] = *reinterpret_cast<const float4*>(src + j);
          x2[it] = *reinterpret_cast<const float4*>(src + half + j);
          if (NS == 2) {
            a1[it] = *reinterpret_cast<const float4*>(src + split_stride + j);
            a2[it] = *reinterpret_cast<const float4*>(src + split_stride + half + j);
          }
          const float4* cs4 = reinterpret_cast<const float4*>(rope_cs + (size_t)pos * half + j);
          ca[it] = cs4[0];
          cb[it] = cs4[1];
        }
      }
#pragma unroll
      for (int it = 0; it < kIt; ++it) {
        const int idx = threadIdx.x + it * blockDim.x;
        if (idx < ntk * g4) {
          const int tt = idx / g4, jg = idx - tt * g4;
          const int t = t0 + tt;
          const int b = t / nq, i = t - b * nq;
          const int pos = bi.len[b] + i;
          float4 u1 = x1[it], u2 = x2[it];
          if (NS == 2) {
            u1.x += a1[it].x; u1.y += a1[it].y; u1.z += a1[it].z; u1.w += a1[it].w;
            u2.x += a2[it].x; u2.y += a2[it].y; u2.z += a2[it].z; u2.w += a2[it].w;
          }
          const float4 c0 = ca[it], c1 = cb[it];  // (cos, sin) of pairs j, j+1 | j+2, j+3
          const float4 r1 = make_float4(u1.x * c0.x - u2.x * c0.y, u1.y * c0.z - u2.y * c0.w,
                                        u1.z * c1.x - u2.z * c1.y, u1.w * c1.z - u2.w * c1.w);
          const float4 r2 = make_float4(u2.x * c0.x + u1.x * c0.y, u2.y * c0.z + u1.y * c0.w,
                                        u2.z * c1.x + u1.z * c1.y, u2.w * c1.z + u1.w * c1.w);
          T* dst = head < hq ? q + (((size_t)b * hq + head) * nq + i) * hd
                             : kc + (((size_t)bi.slot[b] * hkv + (head - hq)) * max_ctx + pos) * hd;
          store4<T>(dst, jg, r1);
          store4<T>(dst + half, jg, r2);
        }
      }
      return;
    }
    T* tile = reinterpret_cast<T*>(rope_smem);
    const int ld = hd + 2;
    const int d4n = hd >> 2;
    constexpr int kItV = 8;   // kRopeTok * 256 / 4 vectors over 256 threads
    float4 xv[kItV], av[kItV];
#pragma unroll
    for (int it = 0; it < kItV; ++it) {
      const int idx = threadIdx.x + it * blockDim.x;
      if (idx < ntk * d4n) {
        const int tt = idx / d4n, jj = (idx - tt * d4n) * 4;
        const float* src = qkv + (size_t)(t0 + tt) * ncol + (size_t)head * hd + jj;
        xv[it] = *reinterpret_cast<const float4*>(src);
        if (NS == 2) av[it] = *reinterpret_cast<const float4*>(src + split_stride);
      }
    }
#pragma unroll
    for (int it = 0; it < kItV; ++it) {
      const int idx = threadIdx.x + it * blockDim.x;
      if (idx < ntk * d4n) {
        const int tt = idx / d4n, jj = (idx - tt * d4n) * 4;
        float4 x = xv[it];
        if (NS == 2) { x.x += av[it].x; x.y += av[it].y; x.z += av[it].z; x.w += av[it].w; }
        T* r = tile + tt * ld + jj;
        r[0] = from_f32<T>(x.x);
        r[1] = from_f32<T>(x.y);
        r[2] = from_f32<T>(x.z);
        r[3] = from_f32<T>(x.w);
      }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (lane < ntk) {
      const int t = t0 + lane;
      const int b = t / nq, i = t - b * nq;
      const int pos = bi.len[b] + i;
      T* col = vt + ((size_t)bi.slot[b] * hkv + (head - hq - hkv)) * hd * (size_t)max_ctx + pos;
      for (int dd = w; dd < hd; dd += nw) col[(size_t)dd * max_ctx] = tile[lane * ld + dd];
    }
    return;
  }
  if (head < hq + hkv) {
    for (int idx = threadIdx.x; idx < ntk * g4; idx += blockDim.x) {
      const int tt = idx / g4, jg = idx - tt * g4, j = jg * 4;
      const int t = t0 + tt;
      const int b = t / nq, i = t - b * nq;
      const int pos = bi.len[b] + i;
      const float* src = qkv + (size_t)t * ncol + (size_t)head * hd;
      float4 x1 = *reinterpret_cast<const float4*>(src + j);
      float4 x2 = *reinterpret_cast<const float4*>(src + half + j);
      for (int sp = 1; sp < nsplit; ++sp) {
        const float4 a = *reinterpret_cast<const float4*>(src + (size_t)sp * split_stride + j);
        const float4 c = *reinterpret_cast<const float4*>(src + (size_t)sp * split_stride + half + j);
        x1.x += a.x; x1.y += a.y; x1.z += a.z; x1.w += a.w;
        x2.x += c.x; x2.y += c.y; x2.z += c.z; x2.w += c.w;
      }
      const float4* cs4 = reinterpret_cast<const float4*>(rope_cs + (size_t)pos * half + j);
      const float4 ca = cs4[0], cb = cs4[1];  // (cos, sin) of pairs j, j+1 | j+2, j+3
      const float4 r1 = make_float4(x1.x * ca.x - x2.x * ca.y, x1.y * ca.z - x2.y * ca.w, x1.z * cb.x - x2.z * cb.y,
                                    x1.w * cb.z - x2.w * cb.w);
      const float4 r2 = make_float4(x2.x * ca.x + x1.x * ca.y, x2.y * ca.z + x1.y * ca.w, x2.z * cb.x + x1.z * cb.y,
                                    x2.w * cb.z + x1.w * cb.w);
      T* dst;
      if (head < hq) {
        dst = q + (((size_t)b * hq + head) * nq + i) * hd;
      } else {
        dst = kc + (((size_t)bi.slot[b] * hkv + (head - hq)) * max_ctx + pos) * hd;
      }
      store4<T>(dst, jg, r1);
      store4<T>(dst + half, jg, r2);
    }
    return;
  }
  T* tile = reinterpret_cast<T*>(rope_smem);
  const int ld = hd + 2;  // odd word stride for 2-byte T: conflict-free column reads
  const int d4n = hd >> 2;
  for (int idx = threadIdx.x; idx < ntk * d4n; idx += blockDim.x) {
    const int tt = idx / d4n, jj = (idx - tt * d4n) * 4;
    const float* src = qkv + (size_t)(t0 + tt) * ncol + (size_t)head * hd + jj;
    float4 x = *reinterpret_cast<const float4*>(src);
    for (int sp = 1; sp < nsplit; ++sp) {
      const float4 a = *reinterpret_cast<const float4*>(src + (size_t)sp * split_stride);
      x.x += a.x; x.y += a.y; x.z += a.z; x.w += a.w;
    }
    T* r = tile + tt * ld + jj;
    r[0] = from_f32<T>(x.x);
    r[1] = from_f32<T>(x.y);
    r[2] = from_f32<T>(x.z);
    r[3] = from_f32<T>(x.w);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane < ntk) {
    const int t = t0 + lane;
    const int b = t / nq, i = t - b * nq;
    const int pos = bi.len[b] + i;
    T* col = vt + ((size_t)bi.slot[b] * hkv + (head - hq - hkv)) * hd * (size_t)max_ctx + pos;
    for (int dd = w; dd < hd; dd += nw) col[(size_t)dd * max_ctx] = tile[lane * ld + dd];
  }
}

template <typename T>
void launch_rope_scatter(const float* qkv, int nsplit, size_t split_stride, T* q, T* kc, T* vt,
                         const float* rope_cs, const BatchInfo& bi, int nq, int hq, int hkv, int hd, int max_ctx,
                         cudaStream_t s) {
  const int n_tok = bi.B * nq;
  if (n_tok <= 0) return;
  if (hd % 8 == 0) {
    dim3 grid((n_tok + kRopeTok - 1) / kRopeTok, hq + 2 * hkv);
    const size_t smem = (size_t)kRopeTok * (hd + 2) * sizeof(T);
    const float2* cs = reinterpret_cast<const float2*>(rope_cs);
    if (hd <= 256 && nsplit == 1)
      launch_k(rope_scatter_tiled_kernel<T, 1>, dim3(grid), dim3(256), smem, s, qkv, nsplit, split_stride, q, kc,
               vt, cs, bi, nq, n_tok, hq, hkv, hd, max_ctx);
    else if (hd <= 256 && nsplit == 2)
      launch_k(rope_scatter_tiled_kernel<T, 2>, dim3(grid), dim3(256), smem, s, qkv, nsplit, split_stride, q, kc,
               vt, cs, bi, nq, n_tok, hq, hkv, hd, max_ctx);
    else
      launch_k(rope_scatter_tiled_kernel<T, 0>, dim3(grid), dim3(256), smem, s, qkv, nsplit, split_stride, q, kc,
               vt, cs, bi, nq, n_tok, hq, hkv, hd, max_ctx);
    return;
  }
  dim3 grid(n_tok, hq + 2 * hkv);
  launch_k(rope_scatter_kernel<T>, dim3(grid), dim3(128), 0, s, qkv, nsplit, split_stride, q, kc, vt,
                                              reinterpret_cast<const float2*>(rope_cs), bi, nq, hq, hkv, hd, max_ctx);
}

// ------------------------------------------------------------ gather rows
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ xn, const int32_t* __restrict__ perm, T* __restrict__ xp,
                                   int k, int d) {
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int src = perm[p] / k;
  // 16-byte vectors when the row is 16-byte aligned (d * sizeof(T) % 16 == 0)
  if ((d * sizeof(T)) % 16 == 0) {
    const int nv = d * (int)sizeof(T) / 16;
    const uint4* s4 = reinterpret_cast<const uint4*>(xn + (size_t)src * d);
    uint4* d4 = reinterpret_cast<uint4*>(xp + (size_t)p * d);
    // four vectors per thread in flight before the first store
    for (int j0 = threadIdx.x; j0 < nv; j0 += 4 * blockDim.x) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u * (int)blockDim.x < nv) r[u] = s4[j0 + u * blockDim.x];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u * (int)blockDim.x < nv) d4[j0 + u * blockDim.x] = r[u];
    }
  } else {
    for (int j = threadIdx.x; j < d; j += blockDim.x) xp[(size_t)p * d + j] = xn[(size_t)src * d + j];
  }
}

template <typename T>
void launch_gather_rows(const T* xn, const int32_t* perm, T* xp, int n_rows, int k, int d, cudaStream_t s) {
  if (n_rows <= 0) return;
  launch_k(gather_rows_kernel<T>, dim3(n_rows), dim3(128), 0, s, xn, perm, xp, k, d);
}

// ------------------------------------------------------------ init canvas
// [P1 一], [P2 运作机制]: the canvas starts as uniform-random vocabulary tokens.
__global__ void init_canvas_kernel(int32_t* canvas, BatchInfo bi, const int* req_ids, int n, int vocab,
                                   uint64_t seed, uint32_t block) {
  pdl_wait();
  pdl_trigger();
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
  launch_k(init_canvas_kernel, dim3(bi.B), dim3(256), 0, s, canvas, bi, req_ids, n, vocab, seed, block);
}

// ----------------------------------------------------------------- set_kv
template <typename T>
__global__ void set_kv_kernel(const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ kc,
                              T* __restrict__ vt, int n, int hd, int max_ctx) {
  pdl_wait();
  pdl_trigger();
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
  launch_k(set_kv_kernel<T>, dim3(dim3(n, hkv)), dim3(128), 0, s, k, v, kc, vt, n, hd, max_ctx);
}

// ----------------------------------------------------------------- get_kv
// Inverse of set_kv: positions [0, n) of one request's cache -> k, v [Hkv, n, hd].
template <typename T>
__global__ void get_kv_kernel(const T* __restrict__ kc, const T* __restrict__ vt, T* __restrict__ k,
                              T* __restrict__ v, int n, int hd, int max_ctx) {
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.y;
  const int p = blockIdx.x;
  for (int j = threadIdx.x; j < hd; j += blockDim.x) {
    k[((size_t)g * n + p) * hd + j] = kc[((size_t)g * max_ctx + p) * hd + j];
    v[((size_t)g * n + p) * hd + j] = vt[((size_t)g * hd + j) * max_ctx + p];
  }
}

template <typename T>
void launch_get_kv(const T* kc, const T* vt, T* k, T* v, int hkv, int n, int hd, int max_ctx, cudaStream_t s) {
  if (n <= 0) return;
  launch_k(get_kv_kernel<T>, dim3(n, hkv), dim3(128), 0, s, kc, vt, k, v, n, hd, max_ctx);
}

// ------------------------------------------------------- wait self-test
// One thread waits on an mbarrier that expects one arrival which never
// comes; the bounded wait gives up after limit_ns and records the code.
__global__ void wait_timeout_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_limit(&bar, 0, err, kErrTimeoutSelftest, limit_ns);
  }
}

void launch_wait_timeout_selftest(int* err, unsigned long long limit_ns, cudaStream_t s) {
  launch_k(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0, s, err, limit_ns);
}

// ------------------------------------------------------------ instantiation
#define DG_INST(T)                                                                                          \
  template void launch_embed<T>(const int32_t*, const int32_t*, const T*, float*, T*, int, int, int, int*,    \
                                cudaStream_t);                                                             \
  template void launch_rmsnorm<T>(const float*, const float*, T*, int, int, float, cudaStream_t);            \
  template void launch_combine<T>(float*, const T*, const float*, int, const float*, T*, int, int, float,     \
                                  cudaStream_t);                                                             \
  template void launch_rope_scatter<T>(const float*, int, size_t, T*, T*, T*, const float*, const BatchInfo&,  \
                                       int, int, int, int, int, cudaStream_t);                               \
  template void launch_add_rmsnorm<T>(float*, const float*, int, size_t, const float*, T*, int, int, float,   \
                                      cudaStream_t);                                                         \
  template void launch_gather_rows<T>(const T*, const int32_t*, T*, int, int, int, cudaStream_t);            \
  template void launch_set_kv<T>(const T*, const T*, T*, T*, int, int, int, int, cudaStream_t);             \
  template void launch_get_kv<T>(const T*, const T*, T*, T*, int, int, int, int, cudaStream_t);
DG_INST(float)
DG_INST(__nv_bfloat16)
#undef DG_INST

}  // namespace dg
