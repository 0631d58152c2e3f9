// Grouped expert GEMMs on CTA pairs (tcgen05 cta_group::2), for the canvas
// step's few tokens per expert ([P1 五]: 256 tokens spread over the experts).
//
// A work item is (expert e, token rows [row0, row0 + rows), 256-row block mb
// of the expert's weights), rows <= 256.  A cluster of two CTAs computes it
// with M = 256: CTA r holds the weight rows mb*256 + 128r .. +127 and half of
// the item's token rows (N/2 of N = 32, 64, 128 or 256 >= rows) in its own
// shared memory; the leader issues the MMAs, which read both CTAs' halves; each CTA's
// TMEM holds its 128 accumulator rows for all N tokens and each CTA writes its
// own output columns.  Per SM and K stage this streams 128 weight rows and
// N/2 token rows, where one CTA per 128-row tile streams all N: an expert's
// token tile crosses each SM half as often.
//   mode 1 (gate/up + SwiGLU): two pair MMAs per K step, the gate and the up
//     rows of the same block into two accumulators; the epilogue writes
//     silu(gate) * up as bf16 rows of the activation [T*k, F].
//   mode 2 (down + scatter): out[row_map[token]] = the bf16 row of d columns
//     (the token-slot order the combine sums in).
// Per CTA, 320 threads: warp 0 lane 0 loads its halves (TMA, 128-byte
// swizzle, completing on the leader's barrier); warp 1 lane 0 of the leader
// issues the MMAs and commits to both CTAs' barriers; warps 2-9 are the
// epilogue, two groups of four warps taking alternate 32-token chunks (each
// staged in shared memory and written as 16-byte row stores), so the
// epilogue keeps up with the main loop at 256-token items.  Each TMA load
// writes only its own CTA's shared memory.  Every wait is bounded; both CTAs
// reach the final cluster barrier before the pair's TMEM is released.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "dg_pair.cuh"
#include "kernels.h"

namespace dg {

namespace {

constexpr int kGM = 128;                 // weight rows per CTA
constexpr int kGK = 64;
constexpr int kGEpiGroups = 2;           // epilogue groups of 4 warps, taking alternate 32-token chunks
constexpr int kGThreads = 64 + kGEpiGroups * 128;
constexpr int kGABytes = kGM * kGK * 2;  // 16 KB: one 64-column chunk of 128 weight rows
constexpr int kGBMaxRows = 128;          // token rows per CTA (the pair's N <= 256)
constexpr int kGMaxSmem = 232448;
constexpr int kGEpiRows = 32;
constexpr int kGEpiBytes = kGEpiRows * kGM * 2;   // bf16 staging tile of one 32-token chunk

struct GPairParams {
  int mode;            // 1 gate/up + SwiGLU, 2 down + scatter
  int M, K;            // weight rows per expert, reduction dim
  int n_mblk;          // 256-row weight blocks per expert
  const int32_t* work;
  const int32_t* n_work;
  __nv_bfloat16* out;
  int ld_out;
  const int32_t* row_map;
  int* err;
  int ksub, stages, stage_bytes, n_a, acc_half, n_acc_buf, acc_cols, tmem_cols;
  int b_rows;          // token rows per CTA a stage has room for (half of the largest N)
  int vec;
};

// Token rows of the pair for an item of `rows` rows: 32, 64, 128 or 256 (each CTA half of it).
__device__ __forceinline__ int pair_n(int rows) {
  return rows <= 32 ? 32 : rows <= 64 ? 64 : rows <= 128 ? 128 : 256;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    gemm_tc2_grouped_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap ta1,
                            const __grid_constant__ CUtensorMap tb16, const __grid_constant__ CUtensorMap tb32,
                            const __grid_constant__ CUtensorMap tb64, const __grid_constant__ CUtensorMap tb128,
                            const GPairParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage0 = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + P.stages * P.stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + P.stages;
  uint64_t* acc_full = bars + 2 * P.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(base + P.stages * P.stage_bytes + 1024);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  int* err = P.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 2 * 4 * kGEpiGroups); }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc2(tmem_slot, (uint32_t)P.tmem_cols);
    tmem_relinquish2();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&ta0);
    if (P.n_a == 2) prefetch_tmap(&ta1);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();             // the work list comes from the launch before
  pdl_trigger();

  const int total = (*P.n_work) * P.n_mblk;
  const int cid = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int nst = (P.K / kGK + P.ksub - 1) / P.ksub;   // stages per item (the last may run past K: zeros)
  const uint32_t a_bytes = (uint32_t)(P.n_a * P.ksub * kGABytes);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    uint32_t kiter = 0;
    bool ok = true;
    for (int item = cid; item < total && ok; item += n_clusters) {
      const int mb = item % P.n_mblk, w = item / P.n_mblk;
      const int e = P.work[3 * w], row0 = P.work[3 * w + 1], rows = P.work[3 * w + 2];
      const int half = pair_n(rows) >> 1;
      const CUtensorMap* tb = half == 16 ? &tb16 : half == 32 ? &tb32 : half == 64 ? &tb64 : &tb128;
      const int m0 = mb * 2 * kGM + (int)rank * kGM;
      const int trow = row0 + (int)rank * half;
      const uint32_t tx = 2u * (a_bytes + (uint32_t)(P.ksub * half * kGK * 2));
      for (int j = 0; j < nst; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
        uint8_t* st = stage0 + (size_t)s * P.stage_bytes;
        const uint32_t fb = map_to_rank(&full[s], 0);   // the leader's barrier counts both CTAs' bytes
        if (leader) mbar_expect_tx(&full[s], tx);
        const int kb0 = j * P.ksub;
        tma_load_4d_pair(st, &ta0, fb, 0, m0, kb0, e);
        if (P.n_a == 2) tma_load_4d_pair(st + P.ksub * kGABytes, &ta1, fb, 0, m0, kb0, e);
        tma_load_3d_pair(st + a_bytes, tb, fb, 0, trow, kb0);
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    uint32_t kiter = 0;
    int it = 0;
    bool ok = true;
    for (int item = cid; item < total && ok; item += n_clusters, ++it) {
      const int w = item / P.n_mblk;
      const int n = pair_n(P.work[3 * w + 2]);
      const int half = n >> 1;
      const uint32_t idesc = idesc_bf16(2 * kGM, n);
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
        for (int c = 0; c < P.ksub; ++c) {
          const uint32_t sa = st + (uint32_t)(c * kGABytes);
          const uint32_t sb = st + a_bytes + (uint32_t)(c * half * kGK * 2);
#pragma unroll
          for (int k = 0; k < kGK / 16; ++k) {
            const uint64_t bdesc = sdesc_k_sw128(sb + 32u * k);
            const uint32_t acc = (j > 0 || c > 0 || k > 0) ? 1u : 0u;
            umma2_bf16(d0, sdesc_k_sw128(sa + 32u * k), bdesc, idesc, acc);
            if (P.n_a == 2)
              umma2_bf16(d0 + (uint32_t)P.acc_half, sdesc_k_sw128(sa + (uint32_t)(P.ksub * kGABytes) + 32u * k),
                         bdesc, idesc, acc);
          }
        }
        umma2_commit_both(&empty[s]);
      }
      if (!ok) break;
      umma2_commit_both(&acc_full[ab]);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Per chunk of 32 tokens: each warp reads its 32-lane quarter of the
    // accumulator (weight row m0 + r, one column per token) into a [token][128]
    // bf16 staging tile; then the 128 threads write whole 256-byte output rows
    // with 16-byte stores.
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const int grp = (warp - 2) >> 2;   // epilogue group
    const int te = threadIdx.x - 64 - 128 * grp;
    __nv_bfloat16* gstg = stg + grp * (kGEpiRows * kGM);
    const uint32_t empty_bar = map_to_rank(&acc_empty[0], 0);
    int it = 0;
    for (int item = cid; item < total; item += n_clusters, ++it) {
      const int mb = item % P.n_mblk, w = item / P.n_mblk;
      const int row0 = P.work[3 * w + 1], rows = P.work[3 * w + 2];
      const int m0 = mb * 2 * kGM + (int)rank * kGM;
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_full[ab], use & 1u, err, kErrTimeoutEpi)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * P.acc_cols);
      for (int c0 = kGEpiRows * grp; c0 < rows; c0 += kGEpiRows * kGEpiGroups) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
        if (P.mode == 1) {
          uint32_t u[32];
          tmem_ld32(tbase + (uint32_t)(P.acc_half + c0), u);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            gstg[j * kGM + r] = __float2bfloat16_rn(
                __fdividef(__uint_as_float(v[j]), 1.f + __expf(-__uint_as_float(v[j]))) * __uint_as_float(u[j]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) gstg[j * kGM + r] = __float2bfloat16_rn(__uint_as_float(v[j]));
        }
        named_barrier_sync(1 + grp, 128);
        const int nrow = min(kGEpiRows, rows - c0);
#pragma unroll 4
        for (int it2 = 0; it2 < kGEpiRows * 16 / 128; ++it2) {
          const int idx = it2 * 128 + te, row = idx >> 4, c8 = idx & 15;
          const int mm = m0 + c8 * 8;
          if (row < nrow && mm < P.M) {
            const int tok = row0 + c0 + row;
            __nv_bfloat16* dst = P.out + (size_t)(P.mode == 2 ? P.row_map[tok] : tok) * P.ld_out + mm;
            const __nv_bfloat16* src = gstg + row * kGM + c8 * 8;
            if (P.vec && mm + 7 < P.M) {
              *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
            } else {
              for (int c = 0; c < 8 && mm + c < P.M; ++c) dst[c] = src[c];
            }
          }
        }
        named_barrier_sync(1 + grp, 128);   // the staging tile is reused by the group's next chunk
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_bar + (uint32_t)(ab * sizeof(uint64_t)));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // the leader's last MMAs have read both CTAs' stages; TMEM is idle
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, (uint32_t)P.tmem_cols);
  }
}

}  // namespace

int launch_gemm_tc2_grouped(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b16,
                            const CUtensorMap& b32, const CUtensorMap& b64, const CUtensorMap& b128, const TcGemm& g,
                            int num_sms, cudaStream_t s) {
  const int ksub = g.ksub >= 1 ? g.ksub : 1;
  if ((g.mode != 1 && g.mode != 2) || g.ntile > 2 * kGBMaxRows || g.K % kGK || (ksub != 1 && ksub != 2))
    return -1;
  GPairParams P{};
  P.mode = g.mode;
  P.M = g.M;
  P.K = g.K;
  P.n_mblk = (g.M + 2 * kGM - 1) / (2 * kGM);
  P.work = g.work;
  P.n_work = g.n_work;
  P.out = reinterpret_cast<__nv_bfloat16*>(g.out);
  P.ld_out = g.ld_out;
  P.row_map = g.row_map;
  P.err = g.err;
  P.ksub = ksub;
  P.n_a = g.mode == 1 ? 2 : 1;
  const int max_n = g.ntile <= 32 ? 32 : g.ntile <= 64 ? 64 : g.ntile <= 128 ? 128 : 256;   // pair_n(ntile)
  P.b_rows = max_n / 2;
  P.acc_half = max_n;                           // the up accumulator's column offset (mode 1)
  P.acc_cols = P.n_a * max_n;                   // columns per accumulator buffer
  P.n_acc_buf = 2 * P.acc_cols <= 512 ? 2 : 1;
  P.tmem_cols = 32;
  while (P.tmem_cols < P.n_acc_buf * P.acc_cols) P.tmem_cols <<= 1;
  if (P.tmem_cols > 512) return -1;
  P.stage_bytes = ksub * (P.n_a * kGABytes + P.b_rows * kGK * 2);
  const int overhead = 1024 + 1024 + kGEpiGroups * kGEpiBytes;
  P.stages = std::min(8, (kGMaxSmem - overhead) / P.stage_bytes);
  if (P.stages < 2) return -1;
  const int smem = overhead + P.stages * P.stage_bytes;
  P.vec = ((uintptr_t)g.out % 16 == 0) && g.ld_out % 8 == 0;
  const int max_items = g.n_work_max * P.n_mblk;
  if (max_items <= 0) return 0;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_tc2_grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGMaxSmem);
    attr = true;
  }
  const int clusters = std::min(max_items, num_sms / 2);
  launch_k(gemm_tc2_grouped_kernel, dim3(2 * clusters), dim3(kGThreads), smem, s, a0, a1, b16, b32, b64, b128, P);
  return 0;
}

}  // namespace dg
