// Grouped expert GEMMs over NVFP4 weights ([P2] 推荐的部署与优化方案, [P4] MoE
// 26B参数架构分析: NVFP4 weights on Blackwell).  Same work items and epilogues
// as the bf16 grouped modes of k_gemm_tc.cu (gate/up with the SwiGLU, down with
// the scatter into token-slot order); the weights arrive as FP4 E2M1 codes with
// E4M3 scales per 16 elements and one fp32 scale per expert matrix.
//
// The activations stay bf16, so the product is the bf16 tensor-core MMA of the
// activations with the dequantised weights: an E2M1 value times an E4M3 value
// has at most 6 significant bits and lies in [2^-10, 2688], so it is exact in
// bf16, and the per-matrix scale is applied to the fp32 accumulator.
//
// 480 threads per CTA:
//   warp 0 lane 0: token producer: the token box (bf16, 128-byte swizzle) of
//     each 64-wide K stage into the stage ring.
//   warp 1 lane 0: tcgen05.mma issuer (M = 128, N = token rows, K = 16).
//   warps 2-5: epilogue (TMEM -> scale by g -> SwiGLU or scatter).
//   warp 6 lane 0: code producer: one TMA box of codes (128 rows x 32 bytes)
//     and one 512-byte bulk copy of their scales (tiled [K/64][rows_pad][4])
//     per weight operand and stage, into a deeper ring of raw slots, so that
//     the HBM reads of the weights run well ahead of the MMA.
//   warps 7-14: dequantisation.  Two threads per tile row expand 32 codes each
//     through a 256-entry table (a code byte -> its two E2M1 values as bf16x2)
//     and one bf16x2 multiply by the block scale, into the 128-byte-swizzled
//     K-major tile the MMA reads; then they free the raw slot and arrive on
//     the stage's full barrier (which also carries the token box's bytes).
// Weight bytes per 128 x 64 tile: 4 KB of codes + 512 B of scales instead of
// 16 KB of bf16.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

namespace {

constexpr int kFBM = 128;
constexpr int kFBK = 64;
constexpr int kFThreads = 480;
constexpr int kDeqThreads = 256;
constexpr int kTileBytes = kFBM * kFBK * 2;   // 16 KB bf16 weight tile
constexpr int kCodeBytes = kFBM * kFBK / 2;   // 4 KB of codes
constexpr int kSfBytes = kFBM * 4;            // 512 B of scales
constexpr int kMaxSmemF = 232448;
constexpr int kEpiRowsF = 32;
constexpr int kRawSlots = 8;

struct Fp4Params {
  int mode;               // 1 gate/up, 2 down
  int M, K, M_pad;        // weight rows per expert, reduction dim, rows padded to 128 (scale tiling)
  int ntile;
  const int32_t* work;
  const int32_t* n_work;
  void* out;
  int ld_out;
  const int32_t* row_map;
  int* err;
  const uint8_t* sf0;     // scales of operand 0 (gate / down)
  const uint8_t* sf1;     // scales of operand 1 (up)
  const float* g0;        // per-expert fp32 scales
  const float* g1;
  int stages, stage_bytes, raw_bytes, acc_cols, n_acc_buf, tmem_cols, n_mtiles, box_levels, vec;
  int off_b;              // byte offset of the token tile inside a stage
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// E2M1 code -> value and E4M3 code -> value (both exact in fp32)
__device__ __forceinline__ float e2m1_f(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const float mag = e == 0 ? 0.5f * (float)m : __int_as_float((int)((e + 126u) << 23 | m << 22));
  return (c & 8u) ? -mag : mag;
}
__device__ __forceinline__ float e4m3_f(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  return e == 0 ? (float)m * 0.001953125f : __int_as_float((int)((e + 120u) << 23 | m << 20));
}

__device__ __forceinline__ int fp4_item_box(const Fp4Params& P, int rows, int* level) {
  int k = 0;
  while (k < P.box_levels && (32 << k) < rows) ++k;
  *level = k;
  return k < P.box_levels ? (32 << k) : P.ntile;
}

__global__ void __launch_bounds__(kFThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tc0, const __grid_constant__ CUtensorMap tc1,
                    const __grid_constant__ CUtensorMap tb, const __grid_constant__ CUtensorMap tbs0,
                    const __grid_constant__ CUtensorMap tbs1, const __grid_constant__ CUtensorMap tbs2,
                    const Fp4Params P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage0 = base;                                         // [stages][stage_bytes]
  uint8_t* raw0 = base + P.stages * P.stage_bytes;                // [kRawSlots][raw_bytes]
  uint32_t* lut = reinterpret_cast<uint32_t*>(raw0 + kRawSlots * P.raw_bytes);   // 256 bf16x2
  uint64_t* bars = reinterpret_cast<uint64_t*>(lut + 256);
  uint64_t* full = bars;                          // token bytes + 256 dequantisation arrivals
  uint64_t* empty = full + P.stages;              // the MMA has read the stage
  uint64_t* raw_full = empty + P.stages;          // codes and scales landed
  uint64_t* raw_empty = raw_full + kRawSlots;     // the dequantisation has read them
  uint64_t* acc_full = raw_empty + kRawSlots;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  __nv_bfloat16* stg_b = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(bars) + 512);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = P.err;
  const int n_a = P.mode == 1 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full[s], 1 + kDeqThreads);
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < kRawSlots; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], kDeqThreads);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
    fence_mbar_init();
  }
  // byte of two E2M1 codes (element 2j low nibble) -> bf16x2 of their values
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(e2m1_f(i & 0xF), e2m1_f(i >> 4));
    lut[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, (uint32_t)P.tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tc0);
    prefetch_tmap(&tb);
    if (P.mode == 1) prefetch_tmap(&tc1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const int total = (*P.n_work) * P.n_mtiles;
  const int nst = P.K / kFBK;
  const int nkc = P.K / kFBK;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ token producer
    uint32_t kiter = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const int w = item / P.n_mtiles;
      const int row0 = P.work[3 * w + 1], rows = P.work[3 * w + 2];
      int lvl;
      const int box = fp4_item_box(P, rows, &lvl);
      const CUtensorMap* bm = box == P.ntile ? &tb : (lvl == 0 ? &tbs0 : lvl == 1 ? &tbs1 : &tbs2);
      for (int j = 0; j < nst; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
        mbar_expect_tx(&full[s], (uint32_t)(box * kFBK * 2));
        tma_load_3d(stage0 + (size_t)s * P.stage_bytes + P.off_b, bm, &full[s], 0, row0, j);
      }
    }
  } else if (warp == 6 && lane == 0) {
    // ------------------------------------------------------------ code producer
    uint32_t kiter = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const int mt = item % P.n_mtiles, w = item / P.n_mtiles;
      const int m0 = mt * kFBM, e = P.work[3 * w];
      for (int j = 0; j < nst; ++j, ++kiter) {
        const int r = kiter % kRawSlots;
        const uint32_t ph = (kiter / kRawSlots) & 1u;
        if (!mbar_wait(&raw_empty[r], ph ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
        uint8_t* rw = raw0 + (size_t)r * P.raw_bytes;
        mbar_expect_tx(&raw_full[r], (uint32_t)(n_a * (kCodeBytes + kSfBytes)));
        tma_load_3d(rw, &tc0, &raw_full[r], j * (kFBK / 2), m0, e);
        bulk_load(rw + n_a * kCodeBytes, P.sf0 + (((size_t)e * nkc + j) * P.M_pad + m0) * 4, kSfBytes, &raw_full[r]);
        if (P.mode == 1) {
          tma_load_3d(rw + kCodeBytes, &tc1, &raw_full[r], j * (kFBK / 2), m0, e);
          bulk_load(rw + 2 * kCodeBytes + kSfBytes, P.sf1 + (((size_t)e * nkc + j) * P.M_pad + m0) * 4, kSfBytes,
                    &raw_full[r]);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t kiter = 0;
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++it) {
      const int w = item / P.n_mtiles;
      const int rows = P.work[3 * w + 2];
      const uint32_t idesc = idesc_bf16(kFBM, (rows + 15) & ~15);
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_empty[ab], (use & 1u) ^ 1u, err, kErrTimeoutMma)) break;
      tc_fence_after();
      const uint32_t d0 = tmem_base + (uint32_t)(ab * P.acc_cols);
      for (int j = 0; j < nst; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        if (!mbar_wait(&full[s], ph, err, kErrTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(stage0 + (size_t)s * P.stage_bytes);
        const uint32_t sb = st + (uint32_t)P.off_b;
#pragma unroll
        for (int k = 0; k < kFBK / 16; ++k) {
          const uint64_t bdesc = sdesc_k_sw128(sb + 32u * k);
          const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
          umma_bf16(d0, sdesc_k_sw128(st + 32u * k), bdesc, idesc, acc);
          if (n_a == 2) umma_bf16(d0 + (uint32_t)P.ntile, sdesc_k_sw128(st + kTileBytes + 32u * k), bdesc, idesc, acc);
        }
        umma_commit(&empty[s]);
      }
      if (!ok) break;
      umma_commit(&acc_full[ab]);
    }
  } else if (warp >= 7) {
    // ------------------------------------------------------------ dequantisation
    const int t = threadIdx.x - 224;                  // 0..255
    const int row = t >> 1, half = t & 1;             // tile row, which 32 of its 64 codes
    const uint32_t r8 = (uint32_t)(row & 7);
    uint32_t kiter = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
      for (int j = 0; j < nst; ++j, ++kiter) {
        const int r = kiter % kRawSlots;
        const int s = kiter % P.stages;
        if (!mbar_wait(&raw_full[r], (kiter / kRawSlots) & 1u, err, kErrTimeoutTma)) { ok = false; break; }
        // the stage's previous contents must have been consumed by the MMA
        if (!mbar_wait(&empty[s], ((kiter / P.stages) & 1u) ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
        const uint8_t* rw = raw0 + (size_t)r * P.raw_bytes;
        uint8_t* st = stage0 + (size_t)s * P.stage_bytes;
        uint4 cw[2];
        uint32_t sfw[2];
        for (int a = 0; a < n_a; ++a) {
          cw[a] = *reinterpret_cast<const uint4*>(rw + a * kCodeBytes + row * 32 + half * 16);
          sfw[a] = *reinterpret_cast<const uint16_t*>(rw + n_a * kCodeBytes + a * kSfBytes + row * 4 + half * 2);
        }
        mbar_arrive(&raw_empty[r]);                    // the raw slot is in registers
        for (int a = 0; a < n_a; ++a) {
          uint8_t* tile = st + a * kTileBytes + (row >> 3) * 1024 + r8 * 128;
          const uint32_t words[4] = {cw[a].x, cw[a].y, cw[a].z, cw[a].w};
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {              // 8 elements: one 16-byte chunk of the bf16 row
            const __nv_bfloat16 sc1 = __float2bfloat16_rn(e4m3_f((sfw[a] >> (8 * (ch >> 1))) & 0xFFu));
            const __nv_bfloat162 sc = __halves2bfloat162(sc1, sc1);
            uint32_t pk[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t v = lut[(words[ch] >> (8 * q)) & 0xFFu];
              const __nv_bfloat162 p2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v), sc);
              pk[q] = *reinterpret_cast<const uint32_t*>(&p2);
            }
            const uint32_t c = (uint32_t)(half * 4 + ch);
            *reinterpret_cast<uint4*>(tile + ((c ^ r8) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&full[s]);
      }
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int te = threadIdx.x - 64;
    __nv_bfloat16* out_b = reinterpret_cast<__nv_bfloat16*>(P.out);
    int it = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
      const int mt = item % P.n_mtiles, w = item / P.n_mtiles;
      const int m0 = mt * kFBM, e = P.work[3 * w], row0 = P.work[3 * w + 1], rows = P.work[3 * w + 2];
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_full[ab], use & 1u, err, kErrTimeoutEpi)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * P.acc_cols);
      const float ga = P.g0[e];
      const float gb = P.mode == 1 ? P.g1[e] : 0.f;
      for (int c0 = 0; c0 < rows; c0 += kEpiRowsF) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
        if (P.mode == 1) {
          // direct form: row m of the SwiGLU output, one token column at a time
          uint32_t u[32];
          tmem_ld32(tbase + (uint32_t)(P.ntile + c0), u);
          const int m = m0 + r;
          if (m < P.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < rows) {
                const float gt = __uint_as_float(v[j]) * ga, up = __uint_as_float(u[j]) * gb;
                out_b[(size_t)(row0 + c0 + j) * P.ld_out + m] =
                    __float2bfloat16_rn(__fdividef(gt, 1.f + __expf(-gt)) * up);
              }
            }
          }
          continue;
        }
        // down: stage the chunk [token][128] and write whole rows through the permutation
#pragma unroll
        for (int j = 0; j < 32; ++j) stg_b[j * kFBM + r] = __float2bfloat16_rn(__uint_as_float(v[j]) * ga);
        named_barrier_sync(1, 128);
        const int nrow = min(kEpiRowsF, rows - c0);
#pragma unroll 4
        for (int it2 = 0; it2 < kEpiRowsF * 16 / 128; ++it2) {
          const int idx = it2 * 128 + te, row = idx >> 4, c8 = idx & 15;
          const int mm = m0 + c8 * 8;
          if (row < nrow && mm < P.M) {
            const int tok = row0 + c0 + row;
            __nv_bfloat16* dst = out_b + (size_t)P.row_map[tok] * P.ld_out + mm;
            const __nv_bfloat16* src = stg_b + row * kFBM + c8 * 8;
            if (P.vec && mm + 7 < P.M) {
              *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
            } else {
              for (int c = 0; c < 8 && mm + c < P.M; ++c) dst[c] = src[c];
            }
          }
        }
        named_barrier_sync(1, 128);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)P.tmem_cols);
  }
}

}  // namespace

int launch_gemm_fp4(const CUtensorMap& c0, const CUtensorMap& c1, const CUtensorMap& b, const CUtensorMap* bsub,
                    const Fp4Gemm& g, int num_sms, cudaStream_t s) {
  Fp4Params P{};
  P.mode = g.mode;
  P.M = g.M;
  P.K = g.K;
  P.M_pad = (g.M + kFBM - 1) / kFBM * kFBM;
  P.ntile = g.ntile;
  P.work = g.work;
  P.n_work = g.n_work;
  P.out = g.out;
  P.ld_out = g.ld_out;
  P.row_map = g.row_map;
  P.err = g.err;
  P.sf0 = g.sf0;
  P.sf1 = g.sf1;
  P.g0 = g.g0;
  P.g1 = g.g1;
  const int n_a = g.mode == 1 ? 2 : 1;
  if (g.K % kFBK || g.ntile < 32 || g.ntile > 256 || g.ntile % 32) return -1;
  P.acc_cols = n_a * g.ntile;
  P.n_acc_buf = 2 * P.acc_cols <= 512 ? 2 : 1;
  P.tmem_cols = 32;
  while (P.tmem_cols < P.n_acc_buf * P.acc_cols) P.tmem_cols <<= 1;
  P.off_b = n_a * kTileBytes;
  P.stage_bytes = (P.off_b + g.ntile * kFBK * 2 + 1023) & ~1023;
  P.raw_bytes = (n_a * (kCodeBytes + kSfBytes) + 1023) & ~1023;
  // LUT 1 KB, barriers and the down projection's staging tile (8 KB) after the rings
  const int overhead = 1024 /*align*/ + 1024 /*lut*/ + 512 /*barriers*/ + kEpiRowsF * kFBM * 2;
  P.stages = std::min(6, (kMaxSmemF - overhead - kRawSlots * P.raw_bytes) / P.stage_bytes);
  if (P.stages < 2) return -1;
  const int smem = overhead + P.stages * P.stage_bytes + kRawSlots * P.raw_bytes;
  P.n_mtiles = (g.M + kFBM - 1) / kFBM;
  P.box_levels = 0;
  if (bsub)
    while (P.box_levels < 3 && (32 << P.box_levels) < g.ntile) ++P.box_levels;
  P.vec = ((uintptr_t)g.out % 16 == 0) && g.ld_out % 8 == 0;
  const int total = g.n_work_max * P.n_mtiles;
  if (total <= 0) return 0;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemF);
    attr = true;
  }
  const int grid = std::min(total, num_sms);
  const CUtensorMap& s0 = P.box_levels > 0 ? bsub[0] : b;
  const CUtensorMap& s1 = P.box_levels > 1 ? bsub[1] : b;
  const CUtensorMap& s2 = P.box_levels > 2 ? bsub[2] : b;
  launch_k(gemm_fp4_kernel, dim3(grid), dim3(kFThreads), smem, s, c0, c1, b, s0, s1, s2, P);
  return 0;
}

}  // namespace dg
