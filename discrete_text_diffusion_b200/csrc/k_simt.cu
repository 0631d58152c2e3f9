// FP32-exact SIMT kernels: the dense GEMM, the grouped expert GEMMs and the
// attention.  They carry the fp32 model end to end (tensor-core fp32 input
// formats round operands to 10-bit mantissas, too coarse for a 1e-4 logit
// match), and they run any dtype, so a bf16 model can use them for shapes the
// tensor-core kernels do not cover.
#include <cuda_bf16.h>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

// ------------------------------------------------------------------- GEMM
// out[t, n] = sum_k x[t, k] * w[n, k]; 64x64 output tile, 16-deep k slices,
// 256 threads with 4x4 outputs each.
constexpr int TS = 64, TK = 16;

template <typename T>
__device__ __forceinline__ void load_tile(const T* __restrict__ src, int rows, int kdim, int r0, int k0,
                                          float (*dst)[TS + 1]) {
  // dst[k][r] = src[(r0 + r) * kdim + k0 + k]
  for (int e = threadIdx.x; e < TS * TK; e += blockDim.x) {
    const int r = e / TK, k = e - r * TK;
    const int gr = r0 + r, gk = k0 + k;
    dst[k][r] = (gr < rows && gk < kdim) ? to_f32(src[(size_t)gr * kdim + gk]) : 0.f;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ x, const T* __restrict__ w, int n_tok,
                                                        int n_out, int kdim, int epi, void* out, int ld_out,
                                                        const float* __restrict__ bias) {
  pdl_wait();
  pdl_trigger();
  __shared__ float xs[TK][TS + 1];
  __shared__ float ws[TK][TS + 1];
  const int t0 = blockIdx.y * TS, n0 = blockIdx.x * TS;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < kdim; k0 += TK) {
    load_tile(x, n_tok, kdim, t0, k0, xs);
    load_tile(w, n_out, kdim, n0, k0, ws);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = xs[k][ty * 4 + i]; b[i] = ws[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= n_tok) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= n_out) continue;
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      const size_t o = (size_t)t * ld_out + n;
      if (epi == EPI_STORE_F32) reinterpret_cast<float*>(out)[o] = v;
      else if (epi == EPI_ADD_F32) reinterpret_cast<float*>(out)[o] += v;
      else reinterpret_cast<T*>(out)[o] = from_f32<T>(v);
    }
  }
}

template <typename T>
void launch_gemm_simt(const T* x, const T* w, int n_tok, int n_out, int kdim, Epi epi, void* out, int ld_out,
                      const float* bias, cudaStream_t s) {
  if (n_tok <= 0 || n_out <= 0) return;
  dim3 grid((n_out + TS - 1) / TS, (n_tok + TS - 1) / TS);
  launch_k(gemm_simt_kernel<T>, dim3(grid), dim3(256), 0, s, x, w, n_tok, n_out, kdim, (int)epi, out, ld_out, bias);
}

// ----------------------------------------------------------- grouped GEMM
// One CTA per (work item, 64-wide output tile).  Work item (e, row0, rows):
// rows [row0, row0+rows) of x belong to expert e (rows <= 64).
template <typename T>
__global__ void __launch_bounds__(256) grouped_simt_kernel(const T* __restrict__ x, const T* __restrict__ wa,
                                                           const T* __restrict__ wb, int n_out, int kdim,
                                                           const int32_t* __restrict__ work,
                                                           const int32_t* __restrict__ n_work,
                                                           const int32_t* __restrict__ perm, int up, void* out,
                                                           int ld_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float xs[TK][TS + 1];
  __shared__ float as[TK][TS + 1];
  __shared__ float bs[TK][TS + 1];
  const int item = blockIdx.y;
  if (item >= *n_work) return;
  const int e = work[3 * item], row0 = work[3 * item + 1], rows = work[3 * item + 2];
  const int n0 = blockIdx.x * TS;
  const T* wae = wa + (size_t)e * n_out * kdim;
  const T* wbe = up ? wb + (size_t)e * n_out * kdim : nullptr;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {}, acc2[4][4] = {};
  for (int k0 = 0; k0 < kdim; k0 += TK) {
    load_tile(x + (size_t)row0 * kdim, rows, kdim, 0, k0, xs);
    load_tile(wae, n_out, kdim, n0, k0, as);
    if (up) load_tile(wbe, n_out, kdim, n0, k0, bs);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4], c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[k][ty * 4 + i];
        b[i] = as[k][tx * 4 + i];
        c[i] = up ? bs[k][tx * 4 + i] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          acc2[i][j] = fmaf(a[i], c[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= n_out) continue;
      if (up) {
        const float g = acc[i][j], u = acc2[i][j];
        const float hv = g / (1.f + expf(-g)) * u;
        reinterpret_cast<T*>(out)[(size_t)(row0 + r) * ld_out + n] = from_f32<T>(hv);
      } else {
        reinterpret_cast<float*>(out)[(size_t)perm[row0 + r] * ld_out + n] = acc[i][j];
      }
    }
  }
}

template <typename T>
void launch_grouped_simt(const T* x, const T* wa, const T* wb, int n_out, int kdim, const int32_t* work,
                         const int32_t* n_work, int n_work_max, const int32_t* perm, bool up, void* out, int ld_out,
                         cudaStream_t s) {
  if (n_work_max <= 0) return;
  dim3 grid((n_out + TS - 1) / TS, n_work_max);
  launch_k(grouped_simt_kernel<T>, dim3(grid), dim3(256), 0, s, x, wa, wb, n_out, kdim, work, n_work, perm, up ? 1 : 0, out, ld_out);
}

// -------------------------------------------------------------- attention
// One CTA of 8 warps handles the same KV head for 8 (query, head) pairs that
// share it (GQA: the r = Hq/Hkv query heads of a KV head).  Keys stream through
// shared memory 32 at a time; lane j scores key j, the warp keeps an online
// softmax, and lane l accumulates output dims l, l+32, ...
// Keys of request b are cache positions [0, len[b] + nq); with causal, query i
// sees keys <= len[b] + i.
constexpr int AW = 8;      // warps per CTA
constexpr int AKT = 32;    // keys per tile
constexpr int AMAXD = 256; // max head dim

template <typename T>
__global__ void __launch_bounds__(AW * 32) attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                                                            const T* __restrict__ vt, T* __restrict__ out,
                                                            AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float smem[];
  const int hd = a.hd, pitch = hd + 1;
  float* ks = smem;                         // [AKT][pitch]
  float* vs = ks + AKT * pitch;             // [AKT][pitch]
  float* qs = vs + AKT * pitch;             // [AW][hd]
  const int r = a.hq / a.hkv;
  const int bg = blockIdx.x;                // b * hkv + g
  const int b = bg / a.hkv, g = bg - b * a.hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = blockIdx.y * (AW / r) + warp / r;  // query index within the request
  const int h = g * r + warp % r;
  const bool active = qi < a.nq;
  const int slot = a.bi.slot[b], plen = a.bi.len[b];
  const int n_keys = plen + a.nq;
  // last query of this CTA bounds the keys it needs
  int kmax = n_keys;
  if (a.causal) {
    const int q_last = min(a.nq - 1, blockIdx.y * (AW / r) + AW / r - 1);
    kmax = min(n_keys, plen + q_last + 1);
  }
  const float scale = rsqrtf((float)hd);
  float* qw = qs + warp * hd;
  if (active) {
    const T* qp = q + (((size_t)b * a.hq + h) * a.nq + qi) * hd;
    for (int d = lane; d < hd; d += 32) qw[d] = to_f32(qp[d]) * scale;
  }
  const T* kbase = kc + ((size_t)slot * a.hkv + g) * a.max_ctx * (size_t)hd;
  const T* vbase = vt + ((size_t)slot * a.hkv + g) * (size_t)hd * a.max_ctx;
  float o[AMAXD / 32];
#pragma unroll
  for (int x = 0; x < AMAXD / 32; ++x) o[x] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int my_lim = a.causal ? plen + qi + 1 : n_keys;
  for (int k0 = 0; k0 < kmax; k0 += AKT) {
    __syncthreads();
    for (int e = threadIdx.x; e < AKT * hd; e += blockDim.x) {
      const int j = e / hd, d = e - j * hd;
      const int key = k0 + j;
      ks[j * pitch + d] = (key < kmax) ? to_f32(kbase[(size_t)key * hd + d]) : 0.f;
    }
    for (int e = threadIdx.x; e < AKT * hd; e += blockDim.x) {
      const int d = e / AKT, j = e - d * AKT;
      const int key = k0 + j;
      vs[j * pitch + d] = (key < kmax) ? to_f32(vbase[(size_t)d * a.max_ctx + key]) : 0.f;
    }
    __syncthreads();
    if (!active) continue;
    const int key = k0 + lane;
    float sc = -INFINITY;
    if (key < my_lim) {
      float acc = 0.f;
      for (int d = 0; d < hd; ++d) acc = fmaf(qw[d], ks[lane * pitch + d], acc);
      sc = acc;
    }
    const float tmax = warp_max(sc);
    const float mn = fmaxf(m, tmax);
    if (mn == -INFINITY) continue;
    const float p = (sc == -INFINITY) ? 0.f : expf(sc - mn);
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int x = 0; x < AMAXD / 32; ++x) o[x] *= corr;
    for (int j = 0; j < AKT; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      if (pj == 0.f) continue;
#pragma unroll
      for (int x = 0; x < AMAXD / 32; ++x) {
        const int d = lane + 32 * x;
        if (d < hd) o[x] = fmaf(pj, vs[j * pitch + d], o[x]);
      }
    }
    m = mn;
  }
  if (!active) return;
  const float inv = 1.f / l;
  T* op = out + ((size_t)b * a.nq + qi) * ((size_t)a.hq * hd) + (size_t)h * hd;
#pragma unroll
  for (int x = 0; x < AMAXD / 32; ++x) {
    const int d = lane + 32 * x;
    if (d < hd) op[d] = from_f32<T>(o[x] * inv);
  }
}

template <typename T>
void launch_attn_simt(const T* q, const T* kc, const T* vt, T* out, const AttnArgs& a, cudaStream_t s) {
  if (a.B <= 0 || a.nq <= 0) return;
  const int r = a.hq / a.hkv;
  const int qpb = AW / r;  // queries per CTA
  dim3 grid(a.B * a.hkv, (a.nq + qpb - 1) / qpb);
  const size_t smem = (size_t)(2 * AKT * (a.hd + 1) + AW * a.hd) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(attn_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    attr_set = true;
  }
  launch_k(attn_simt_kernel<T>, dim3(grid), dim3(AW * 32), smem, s, q, kc, vt, out, a);
}

#define DG_INST(T)                                                                                           \
  template void launch_gemm_simt<T>(const T*, const T*, int, int, int, Epi, void*, int, const float*,         \
                                    cudaStream_t);                                                            \
  template void launch_grouped_simt<T>(const T*, const T*, const T*, int, int, const int32_t*, const int32_t*, \
                                       int, const int32_t*, bool, void*, int, cudaStream_t);                  \
  template void launch_attn_simt<T>(const T*, const T*, const T*, T*, const AttnArgs&, cudaStream_t);
DG_INST(float)
DG_INST(__nv_bfloat16)
#undef DG_INST

}  // namespace dg
