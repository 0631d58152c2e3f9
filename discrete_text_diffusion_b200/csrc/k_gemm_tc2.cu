// Dense tensor-core GEMM on CTA pairs (tcgen05 cta_group::2), for the split-K
// projections of a canvas step: out[token, m] = sum_k W[m, k] * X[token, k].
//
// A cluster of two CTAs on neighbouring SMs computes one 256-row weight tile
// against a token tile of N rows: CTA r holds weight rows m0 + 128 r (the M
// half of the MMA's A operand) and token rows row0 + r N/2 (the N half of its
// B operand) in its own shared memory, and the pair's leader issues
// tcgen05.mma.cta_group::2 with M = 256.  Each SM therefore streams 128 weight
// rows and only half of the token tile per K stage; at 256 tokens the token
// operand is as large as the weights, so this cuts each SM's operand ingest by
// a third against one CTA per 128-row tile.  The accumulator is split the
// same way: CTA r's TMEM holds its 128 rows for all N tokens, and each CTA runs
// the epilogue of its own rows.
//
// Per CTA, 192 threads: warp 0 lane 0 loads its halves (TMA, 128-byte swizzle,
// completing on the leader's full barrier); warp 1 lane 0 of the leader issues
// the MMAs and commits to both CTAs' barriers; warps 2-5 are the epilogue
// (fp32 partial slices through TMA stores, or plain stores).  The epilogues of
// both CTAs free an accumulator buffer by arriving on the leader's barrier.
// Each TMA load writes only its own CTA's shared memory.  Every wait is
// bounded; a CTA that gives up still reaches the final cluster barrier, so
// neither CTA leaves while the other may read its shared memory.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "dg_pair.cuh"
#include "kernels.h"

namespace dg {

namespace {

constexpr int kPM = 128;              // weight rows per CTA (the pair's tile is 256)
constexpr int kPK = 64;
constexpr int kPThreads = 192;
constexpr int kPABytes = kPM * kPK * 2;   // 16 KB
constexpr int kPMaxSmem = 232448;
constexpr int kPEpiRows = 32;
constexpr int kPEpiBytes = kPEpiRows * kPM * 4;   // 16 KB staging tile (fp32)

struct PairParams {
  int M, K, T;
  int ntile;          // token rows of the pair's tile (each CTA holds ntile / 2)
  int seg1, seg2;     // first weight row served by map a1 / a2 (multiples of 256)
  int ksplit;
  size_t split_stride;
  float* out;
  int ld_out;
  int* err;
  int ksub;           // 64-column chunks per stage (one TMA instruction per operand)
  int stages, stage_bytes, acc_cols, n_acc_buf, tmem_cols, n_mpairs, n_ttiles;
  int tma_out, vec;
};

__device__ __forceinline__ void pair_item(const PairParams& P, int item, int nst, int rank, int& m0, int& row0,
                                          int& rows_pair, int& j0, int& j1, int& ks) {
  const int nsplit = P.ksplit > 1 ? P.ksplit : 1;
  ks = item % nsplit;
  const int rest = item / nsplit;
  const int tt = rest % P.n_ttiles, mp = rest / P.n_ttiles;
  m0 = mp * 2 * kPM + rank * kPM;
  const int r0 = tt * P.ntile;
  rows_pair = min(P.ntile, P.T - r0);
  row0 = r0 + rank * (P.ntile / 2);
  j0 = ks * nst / nsplit;
  j1 = (ks + 1) * nst / nsplit;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap ta1,
                    const __grid_constant__ CUtensorMap ta2, const __grid_constant__ CUtensorMap tb,
                    const __grid_constant__ CUtensorMap tout, const PairParams P) {
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
  float* stg = reinterpret_cast<float*>(base + P.stages * P.stage_bytes + 1024);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  int* err = P.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 2 * 128); }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc2(tmem_slot, (uint32_t)P.tmem_cols);
    tmem_relinquish2();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&ta0);
    prefetch_tmap(&tb);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the producer waits for the previous launch only after its first weight boxes
  if (!(warp == 0 && lane == 0)) pdl_wait();
  pdl_trigger();

  const int n_items = P.n_mpairs * P.n_ttiles * (P.ksplit > 1 ? P.ksplit : 1);
  const int cid = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int nst = (P.K / kPK + P.ksub - 1) / P.ksub;   // stages of ksub chunks (the last may run past K: zeros)
  const int bhalf = P.ntile / 2;                 // token rows this CTA holds
  const uint32_t a_bytes = (uint32_t)(P.ksub * kPABytes);
  const uint32_t b_chunk = (uint32_t)(bhalf * kPK * 2);
  const uint32_t b_bytes = (uint32_t)P.ksub * b_chunk;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // The weights are never written by the launch just before this one: the
    // first item's first stages (free, the ring is empty) receive their
    // weight boxes before the wait for that launch; the token boxes after it.
    auto weight_map = [&](int m0, int& am0) -> const CUtensorMap* {
      const int mp0 = m0 - (int)rank * kPM;
      if (mp0 >= P.seg2) { am0 = m0 - P.seg2; return &ta2; }
      if (mp0 >= P.seg1) { am0 = m0 - P.seg1; return &ta1; }
      am0 = m0;
      return &ta0;
    };
    int pre = 0;
    if (cid < n_items) {
      int m0, row0, rows_pair, j0, j1, ks, am0;
      pair_item(P, cid, nst, (int)rank, m0, row0, rows_pair, j0, j1, ks);
      const CUtensorMap* am = weight_map(m0, am0);
      pre = min(P.stages, j1 - j0);
      for (int i = 0; i < pre; ++i) {
        if (leader) mbar_expect_tx(&full[i], 2u * (a_bytes + b_bytes));
        tma_load_3d_pair(stage0 + (size_t)i * P.stage_bytes, am, map_to_rank(&full[i], 0), 0, am0,
                         (j0 + i) * P.ksub);
      }
    }
    pdl_wait();
    uint32_t kiter = 0;
    bool ok = true;
    for (int item = cid; item < n_items && ok; item += n_clusters) {
      int m0, row0, rows_pair, j0, j1, ks, am0;
      pair_item(P, item, nst, (int)rank, m0, row0, rows_pair, j0, j1, ks);
      const CUtensorMap* am = weight_map(m0, am0);
      for (int j = j0; j < j1; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        uint8_t* st = stage0 + (size_t)s * P.stage_bytes;
        const uint32_t fb = map_to_rank(&full[s], 0);   // the leader's barrier counts both CTAs' bytes
        if (kiter >= (uint32_t)pre) {
          if (!mbar_wait(&empty[s], ph ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
          if (leader) mbar_expect_tx(&full[s], 2u * (a_bytes + b_bytes));
          tma_load_3d_pair(st, am, fb, 0, am0, j * P.ksub);
        }
        tma_load_3d_pair(st + a_bytes, &tb, fb, 0, row0, j * P.ksub);
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    uint32_t kiter = 0;
    int it = 0;
    bool ok = true;
    const uint32_t idesc = idesc_bf16(2 * kPM, P.ntile);
    for (int item = cid; item < n_items && ok; item += n_clusters, ++it) {
      int m0, row0, rows_pair, j0, j1, ks;
      pair_item(P, item, nst, 0, m0, row0, rows_pair, j0, j1, ks);
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_empty[ab], (use & 1u) ^ 1u, err, kErrTimeoutMma)) break;
      tc_fence_after();
      const uint32_t d0 = tmem_base + (uint32_t)(ab * P.acc_cols);
      for (int j = j0; j < j1; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        if (!mbar_wait(&full[s], ph, err, kErrTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(stage0 + (size_t)s * P.stage_bytes);
        for (int c = 0; c < P.ksub; ++c)
#pragma unroll
          for (int k = 0; k < kPK / 16; ++k)
            umma2_bf16(d0, sdesc_k_sw128(st + (uint32_t)c * kPABytes + 32u * k),
                       sdesc_k_sw128(st + a_bytes + (uint32_t)c * b_chunk + 32u * k), idesc,
                       (j > j0 || c > 0 || k > 0) ? 1u : 0u);
        umma2_commit_both(&empty[s]);
      }
      if (!ok) break;
      umma2_commit_both(&acc_full[ab]);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int te = threadIdx.x - 64;
    const uint32_t empty_bar = map_to_rank(&acc_empty[0], 0);
    uint32_t chunk_no = 0;
    int it = 0;
    for (int item = cid; item < n_items; item += n_clusters, ++it) {
      int m0, row0, rows_pair, j0, j1, ks;
      pair_item(P, item, nst, (int)rank, m0, row0, rows_pair, j0, j1, ks);
      const int row_pair0 = row0 - (int)rank * bhalf;    // the pair's first token row: TMEM column 0
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_full[ab], use & 1u, err, kErrTimeoutEpi)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * P.acc_cols);
      for (int c0 = 0; c0 < rows_pair; c0 += kPEpiRows) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
        if (P.tma_out) {
          float* tile = stg + (chunk_no & 1u) * (kPEpiBytes / 4);
          if (te == 0 && chunk_no >= 2) bulk_wait_read_1();
          named_barrier_sync(1, 128);
#pragma unroll
          for (int j = 0; j < 32; ++j) tile[j * kPM + r] = __uint_as_float(v[j]);
          fence_proxy_async_smem();
          named_barrier_sync(1, 128);
          if (te == 0) {
            tma_store_3d(&tout, tile, m0, row_pair0 + c0, ks);
            bulk_commit();
          }
          ++chunk_no;
          continue;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) stg[j * kPM + r] = __uint_as_float(v[j]);
        named_barrier_sync(1, 128);
        const int nrow = min(kPEpiRows, rows_pair - c0);
#pragma unroll 4
        for (int it2 = 0; it2 < kPEpiRows * 32 / 128; ++it2) {
          const int idx = it2 * 128 + te, row = idx >> 5, c4 = idx & 31;
          const int mm = m0 + c4 * 4;
          if (row < nrow && mm < P.M) {
            float* dst = P.out + (size_t)ks * P.split_stride + (size_t)(row_pair0 + c0 + row) * P.ld_out + mm;
            const float4 val = *reinterpret_cast<const float4*>(stg + row * kPM + c4 * 4);
            if (P.vec && mm + 3 < P.M) {
              *reinterpret_cast<float4*>(dst) = val;
            } else {
              const float vv[4] = {val.x, val.y, val.z, val.w};
              for (int c = 0; c < 4 && mm + c < P.M; ++c) dst[c] = vv[c];
            }
          }
        }
        named_barrier_sync(1, 128);
      }
      tc_fence_before();
      mbar_arrive_cluster(empty_bar + (uint32_t)(ab * sizeof(uint64_t)));
    }
    if (P.tma_out && te == 0) bulk_wait_read_all();
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

int launch_gemm_tc_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b,
                        const TcGemm& g, int num_sms, cudaStream_t s, const CUtensorMap* tout) {
  const int ksub = g.ksub >= 1 ? g.ksub : 1;
  if (g.mode != 0 || g.ntile < 32 || g.ntile > 256 || g.ntile % 32 || g.K % kPK || (ksub != 1 && ksub != 2 && ksub != 4))
    return -1;
  if (g.ksplit > (g.K / kPK + ksub - 1) / ksub) return -1;
  if ((g.seg1 != INT_MAX && g.seg1 % (2 * kPM)) || (g.seg2 != INT_MAX && g.seg2 % (2 * kPM))) return -1;
  PairParams P{};
  P.M = g.M;
  P.K = g.K;
  P.T = g.T;
  P.ntile = g.ntile;
  P.seg1 = g.seg1;
  P.seg2 = g.seg2;
  P.ksplit = g.ksplit > 1 ? g.ksplit : 1;
  P.split_stride = g.split_stride;
  P.out = reinterpret_cast<float*>(g.out);
  P.ld_out = g.ld_out;
  P.err = g.err;
  P.acc_cols = g.ntile;
  P.n_acc_buf = 2 * P.acc_cols <= 512 ? 2 : 1;
  P.tmem_cols = 32;
  while (P.tmem_cols < P.n_acc_buf * P.acc_cols) P.tmem_cols <<= 1;
  P.ksub = ksub;
  P.stage_bytes = ksub * (kPABytes + (g.ntile / 2) * kPK * 2);
  P.tma_out = tout != nullptr;
  const int overhead = 1024 + 1024 + (P.tma_out ? 2 : 1) * kPEpiBytes;
  P.stages = std::min(8, (kPMaxSmem - overhead) / P.stage_bytes);
  if (P.stages < 2) return -1;
  const int smem = overhead + P.stages * P.stage_bytes;
  P.n_mpairs = (g.M + 2 * kPM - 1) / (2 * kPM);
  P.n_ttiles = (g.T + g.ntile - 1) / g.ntile;
  P.vec = ((uintptr_t)g.out % 16 == 0) && g.ld_out % 4 == 0 && (P.ksplit <= 1 || g.split_stride % 4 == 0);
  const int n_items = P.n_mpairs * P.n_ttiles * P.ksplit;
  if (n_items <= 0) return 0;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPMaxSmem);
    attr = true;
  }
  const int clusters = std::min(n_items, num_sms / 2);
  launch_k(gemm_tc2_kernel, dim3(2 * clusters), dim3(kPThreads), smem, s, a0, a1, a2, b, tout ? *tout : b, P);
  return 0;
}

}  // namespace dg
