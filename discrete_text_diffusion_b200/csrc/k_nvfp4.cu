// NVFP4 expert weights ([P2] 推荐的部署与优化方案, [P4] MoE 26B参数架构分析: the
// model is deployed with NVFP4 weights on Blackwell).  Element codes are FP4
// E2M1 (OCP Microscaling spec: 1 sign, 2 exponent bits with bias 1, 1 mantissa
// bit, largest magnitude 6); block scales are E4M3 (OCP OFP8: 4 exponent bits
// with bias 7, 3 mantissa bits, largest finite 448), one per 16 consecutive
// elements along the contraction dimension; one fp32 scale g per matrix.
//
// This file holds the device quantiser (dg_quantize_nvfp4).  The storage it
// writes is the one the expert GEMM reads: codes row-major with element 2j in
// the low nibble of byte j; block scales tiled [K/64][rows_pad][4] so that the
// 128 rows x 4 scales of one 64-wide K chunk are 512 contiguous bytes.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "dg.h"
#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

namespace {

constexpr double kE2M1Max = 6.0;
constexpr double kE4M3Max = 448.0;

// E4M3 code -> value (codes 0..0x7E; 0x7F is NaN and never produced here)
__device__ __forceinline__ double e4m3_value(uint32_t c) {
  const int e = (c >> 3) & 0xF, m = c & 7;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
  return (c & 0x80) ? -mag : mag;
}

// Non-negative x -> E4M3 code: nearest value, ties to the even code, x >= 448
// saturates to 448.  Inside a binade the values are evenly spaced and the code
// parity is the parity of the step count, so this is round-half-even of x / step.
__device__ __forceinline__ uint32_t e4m3_encode_nonneg(double x) {
  if (!(x > 0.0)) return 0u;
  if (x >= kE4M3Max) return 0x7Eu;
  if (x < 0.015625) return (uint32_t)rint(x * 512.0);   // below 2^-6: step 2^-9 (8 steps -> code 8 = 2^-6)
  int ex;
  frexp(x, &ex);                                         // x in [2^(ex-1), 2^ex)
  const int E = ex - 1;
  const double q = rint(ldexp(x, 3 - E));               // in [8, 16]
  return (uint32_t)((E + 7) * 8 + (int)q - 8);           // q = 16 rolls into the next binade
}

// y -> E2M1 code: nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6 with ties to the even
// code, saturating at 6; the sign bit follows the sign of y.
__device__ __forceinline__ uint32_t e2m1_encode(double y) {
  const double a = fabs(y);
  uint32_t c;
  if (a <= 0.25) c = 0;
  else if (a < 0.75) c = 1;
  else if (a <= 1.25) c = 2;
  else if (a < 1.75) c = 3;
  else if (a <= 2.5) c = 4;
  else if (a < 3.5) c = 5;
  else if (a <= 5.0) c = 6;
  else c = 7;
  return c | (signbit(y) ? 0x8u : 0u);
}

__global__ void nvfp4_amax_kernel(const __nv_bfloat16* __restrict__ w, size_t per_mat, unsigned* __restrict__ amax_bits) {
  const int mat = blockIdx.y;
  const __nv_bfloat16* p = w + (size_t)mat * per_mat;
  float m = 0.f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_mat; i += (size_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(p[i])));
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[mat], __float_as_uint(m));   // non-negative floats order as integers
}

__global__ void nvfp4_zero_kernel(unsigned* __restrict__ x, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) x[i] = 0u;
}

// in place: amax bits -> g = fp32(amax / (6 * 448)), 1 for an all-zero matrix
__global__ void nvfp4_global_scale_kernel(float* __restrict__ g, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float amax = __uint_as_float(reinterpret_cast<unsigned*>(g)[i]);
  g[i] = amax > 0.f ? (float)((double)amax / (kE2M1Max * kE4M3Max)) : 1.f;
}

// one thread per 16-element block; threads past the rows write the padding rows' zero scales
__global__ void nvfp4_encode_kernel(const __nv_bfloat16* __restrict__ w, int n_mats, int rows, int rows_pad, int K,
                                    const float* __restrict__ g, uint8_t* __restrict__ codes,
                                    uint8_t* __restrict__ scales) {
  const int nb = K / 16;
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t total = (size_t)n_mats * rows_pad * nb;
  if (idx >= total) return;
  const int blk = (int)(idx % nb);
  const int row = (int)((idx / nb) % rows_pad);
  const int mat = (int)(idx / ((size_t)nb * rows_pad));
  uint8_t* sc = scales + ((size_t)mat * (K / 64) + blk / 4) * rows_pad * 4 + (size_t)row * 4 + (blk & 3);
  if (row >= rows) {
    *sc = 0;
    return;
  }
  const __nv_bfloat16* src = w + ((size_t)mat * rows + row) * K + (size_t)blk * 16;
  float x[16];
  double amax_b = 0.0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    x[i] = __bfloat162float(src[i]);
    amax_b = fmax(amax_b, (double)fabsf(x[i]));
  }
  const double gd = (double)g[mat];
  const uint32_t s_code = e4m3_encode_nonneg(amax_b / (kE2M1Max * gd));
  const double s_val = e4m3_value(s_code);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = s_val > 0.0 ? e2m1_encode((double)x[i] / (s_val * gd)) : 0u;
    if (i < 8) lo |= q << (4 * i);
    else hi |= q << (4 * (i - 8));
  }
  *sc = (uint8_t)s_code;
  *reinterpret_cast<uint2*>(codes + ((size_t)mat * rows + row) * (K / 2) + (size_t)blk * 8) = make_uint2(lo, hi);
}

int report(char* err, size_t err_len, int code, const char* fmt, ...) {
  if (err && err_len > 0) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(err, err_len, fmt, ap);
    va_end(ap);
  }
  return code;
}

}  // namespace

}  // namespace dg

using namespace dg;

extern "C" int dg_quantize_nvfp4(const void* w, int n_mats, int rows, int K, uint8_t* codes, uint8_t* scales,
                                 float* g, void* stream, char* err, size_t err_len) {
  if (err && err_len > 0) err[0] = '\0';
  if (!w || !codes || !scales || !g) return report(err, err_len, DG_EINVAL, "null pointer");
  if (n_mats < 1 || rows < 1 || K < 64 || K % 64) return report(err, err_len, DG_EINVAL, "bad shape: n_mats >= 1, rows >= 1, K a multiple of 64");
  if (((uintptr_t)w & 15u) || ((uintptr_t)codes & 15u))
    return report(err, err_len, DG_EINVAL, "w and codes must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows_pad = (rows + 127) / 128 * 128;
  const size_t per_mat = (size_t)rows * K;
  nvfp4_zero_kernel<<<(n_mats + 255) / 256, 256, 0, s>>>(reinterpret_cast<unsigned*>(g), n_mats);
  const int bx = (int)std::min<size_t>(64, (per_mat + 256 * 16 - 1) / (256 * 16));
  nvfp4_amax_kernel<<<dim3(bx, n_mats), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), per_mat,
                                                      reinterpret_cast<unsigned*>(g));
  nvfp4_global_scale_kernel<<<(n_mats + 255) / 256, 256, 0, s>>>(g, n_mats);
  const size_t total = (size_t)n_mats * rows_pad * (K / 16);
  nvfp4_encode_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), n_mats,
                                                                     rows, rows_pad, K, g, codes, scales);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return report(err, err_len, DG_ECUDA, "quantiser launch: %s", cudaGetErrorString(e));
  return DG_OK;
}
