// tcgen05 GEMM for the bf16 model: out[token, m] = sum_k W[m, k] * X[token, k].
//
// The weight matrix is the 128-row M operand and the tokens are the N
// operand (N = 32..256 per tile).  A canvas step has few tokens per expert
// ([P1 五]: 256 tokens spread over ~84-128 experts), so putting the weights on
// the M side keeps the tensor-core tile full while each weight tile streams
// from HBM once per token tile.
//
// Persistent kernel, 192 threads:
//   warp 0  lane 0: TMA producer (weights 128x64 + tokens Nx64 per stage,
//           128-byte swizzle) into a ring of shared-memory stages
//   warp 1  lane 0: issues tcgen05.mma (M=128, N, K=16) into a TMEM
//           accumulator; tcgen05.commit frees stages / signals the epilogue
//   warps 2-5: epilogue, each reading its 32-lane quarter of TMEM
// Accumulators are double-buffered in TMEM when they fit, so the epilogue of
// one tile overlaps the main loop of the next.
//
// Modes:
//   0 dense: up to three weight maps stacked along M (the Q | K | V
//     projections); epilogue store fp32, add fp32 (residual), or store bf16.
//   1 grouped up: per work item (expert e, row0, rows) the gate and the up
//     weights of expert e both multiply the same token tile into two
//     accumulators; the epilogue writes silu(gate) * up as bf16.
//   2 grouped down: expert e's down projection; the epilogue writes row r to
//     out[row_map[r]] (the token-slot order) as bf16 (the combine adds the
//     slots in fp32).
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kBoxN = 32;
constexpr int kTcThreads = 192;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kMaxSmem = 232448;        // 227 KB opt-in limit per CTA
#ifndef DG_GEMM_MAX_STAGES
#define DG_GEMM_MAX_STAGES 8            // shared-memory pipeline depth cap
#endif
#ifndef DG_GEMM_KSUB
#define DG_GEMM_KSUB 1                  // default 64-wide K blocks per stage
#endif
#ifndef DG_GEMM_CTAS_PER_SM
#define DG_GEMM_CTAS_PER_SM 1           // default co-resident CTAs per SM
#endif
constexpr int kSmemPerSm = 233472;      // 228 KB of shared memory per SM
#ifndef DG_EPI_STAGE_MODES
#define DG_EPI_STAGE_MODES 5            // bit m: mode m writes its output through the staging tile (dense and
                                        // expert down; the bf16 gate/up output measured a loss)
#endif
constexpr int kEpiRows = 32;            // token rows per epilogue chunk
constexpr int kEpiBytes = kEpiRows * kBM * 4;  // staging tile of one chunk (fp32) = 16 KB

struct TcLayout {
  int n_a;          // weight operands per stage (1 or 2)
  int ksub;         // 64-wide K blocks per stage
  int stage_bytes;
  int stages;
  int acc_cols;     // TMEM columns of one accumulator buffer (all operands)
  int n_acc_buf;
  int tmem_cols;    // power of two >= 32
  int smem_bytes;
  int per_sm;       // CTAs per SM the grid is sized for
};

static TcLayout tc_layout(const TcGemm& p) {
  TcLayout L;
  L.n_a = (p.mode == 1) ? 2 : 1;
  L.acc_cols = L.n_a * p.ntile;
  L.per_sm = std::max(1, std::min(3, p.ctas_per_sm > 0 ? p.ctas_per_sm : DG_GEMM_CTAS_PER_SM));
  // the tensor maps are built for this chunk count: it is never changed here
  L.ksub = std::max(1, std::min(4, p.ksub > 0 ? p.ksub : DG_GEMM_KSUB));
  const int n_stg = ((DG_EPI_STAGE_MODES >> p.mode) & 1) ? (p.tma_out ? 2 : 1) : 0;   // staging tiles
  const int overhead = 1024 /*align*/ + 1024 /*barriers*/ + n_stg * kEpiBytes;
  for (;;) {
    // TMEM: every co-resident CTA holds its accumulators
    L.n_acc_buf = (L.per_sm * 2 * L.acc_cols <= 512) ? 2 : 1;
    const int need = L.n_acc_buf * L.acc_cols;
    L.tmem_cols = 32;
    while (L.tmem_cols < need) L.tmem_cols <<= 1;
    const int budget = std::min(kMaxSmem, kSmemPerSm / L.per_sm - 1024);
    L.stage_bytes = L.ksub * (L.n_a * kABytes + p.ntile * kBK * 2);
    L.stages = std::min(DG_GEMM_MAX_STAGES, (budget - overhead) / L.stage_bytes);
    if (L.per_sm * L.tmem_cols <= 512 && L.stages >= 2) break;
    if (L.per_sm > 1) { --L.per_sm; continue; }
    break;   // stages < 2: rejected by the launcher
  }
  L.smem_bytes = overhead + L.stages * L.stage_bytes;
  return L;
}

int gemm_tc_smem_bytes(const TcGemm& p, int* stages) {
  TcLayout L = tc_layout(p);
  if (stages) *stages = L.stages;
  return L.smem_bytes;
}

// silu(g) * u for an output rounded to bf16 right after: the hardware exp2
// and the approximate divide (their few-ulp error is far below bf16's 2^-9).
__device__ __forceinline__ float swiglu_bf16(float gt, float up) {
  return __fdividef(gt, 1.f + __expf(-gt)) * up;
}

struct TcKParams {
  TcGemm g;
  int stages, stage_bytes, acc_cols, n_acc_buf, tmem_cols, n_mtiles, n_ttiles, ksub;
  int vec;         // output rows may be written as aligned 16-byte vectors
  int box_levels;  // grouped modes: token maps tbs[k] with boxes of 32 << k rows (< ntile) exist for k < box_levels
};

// Token box of a work item: grouped modes load only as many rows as the item
// has (a box of 32, 64, 128, ... rows, at most ntile); dense mode always ntile.
__device__ __forceinline__ int item_box(const TcKParams& P, int rows, int* level) {
  int k = 0;
  if (P.g.mode != 0)
    while (k < P.box_levels && (32 << k) < rows) ++k;
  *level = k;
  return k < P.box_levels ? (32 << k) : P.g.ntile;
}

// Work item -> weight tile, token rows and (dense split-K) the range of K
// stages [j0, j1) with its split index ks.
__device__ __forceinline__ void tc_item(const TcKParams& P, int item, int nst, int& m0, int& e, int& row0,
                                        int& rows, int& j0, int& j1, int& ks) {
  const TcGemm& g = P.g;
  j0 = 0;
  j1 = nst;
  ks = 0;
  if (g.mode == 0) {
    const int nsplit = g.ksplit > 1 ? g.ksplit : 1;
    ks = item % nsplit;
    const int rest = item / nsplit;
    const int tt = rest % P.n_ttiles, mt = rest / P.n_ttiles;
    m0 = mt * kBM;
    e = 0;
    row0 = tt * g.ntile;
    rows = min(g.ntile, g.T - row0);
    j0 = ks * nst / nsplit;
    j1 = (ks + 1) * nst / nsplit;
  } else {
    const int mt = item % P.n_mtiles, w = item / P.n_mtiles;
    m0 = mt * kBM;
    e = g.work[3 * w];
    row0 = g.work[3 * w + 1];
    rows = g.work[3 * w + 2];
  }
}

// kStats: the LM head's sampler-statistics epilogue (EPI_VOCAB_STATS), compiled
// as its own instantiation so that its registers do not weigh on the other modes.
template <bool kStats>
__global__ void __launch_bounds__(kTcThreads, 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap ta1,
                   const __grid_constant__ CUtensorMap ta2, const __grid_constant__ CUtensorMap tb,
                   const __grid_constant__ CUtensorMap tbs0, const __grid_constant__ CUtensorMap tbs1,
                   const __grid_constant__ CUtensorMap tbs2, const __grid_constant__ CUtensorMap tout,
                   const TcKParams P) {
  extern __shared__ uint8_t smem_raw[];
  const TcGemm& g = P.g;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage0 = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + P.stages * P.stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + P.stages;
  uint64_t* acc_full = bars + 2 * P.stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = g.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, (uint32_t)P.tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&ta0);
    prefetch_tmap(&tb);
    if (g.mode == 1) prefetch_tmap(&ta1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above touches no global memory: it overlaps the previous
  // kernel.  So does the dense producer's first weight boxes (below): dense
  // weights are never written by the launch just before this one.
  const bool prefetch_a = g.mode == 0;
  if (!(prefetch_a && warp == 0 && lane == 0)) pdl_wait();
  pdl_trigger();

  // (the prefetching producer has not waited yet; mode 0 reads no n_work)
  const int total = (g.mode == 0) ? P.n_mtiles * P.n_ttiles * (g.ksplit > 1 ? g.ksplit : 1)
                                  : (*g.n_work) * P.n_mtiles;
  const int nk = g.K / kBK;                       // 64-wide K blocks
  const int ksub = P.ksub;                        // K blocks per pipeline stage
  const int nst = (nk + ksub - 1) / ksub;         // stages per output tile
  const int n_a = (g.mode == 1) ? 2 : 1;
  // stage layout: [ksub x A0][ksub x A1 (mode 1)][ksub x B], each sub 1024-aligned

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // One TMA instruction per operand and stage: the weight maps are
    // (64, rows, K/64[, experts]) views with a box of ksub 64-column chunks,
    // the token map a (64, rows, K/64) view with a box of ntile rows x ksub
    // chunks.  A stage always receives whole boxes (chunks past K, rows past
    // the matrix are zero-filled), so the byte count is fixed.
    // Dense mode: the weight boxes of the first item's first stages go out
    // before waiting for the previous launch (the ring is empty, so those
    // stages are free); the token boxes follow once it has finished.
    int pre = 0;
    if (prefetch_a) {
      if ((int)blockIdx.x < total) {
        int m0, e, row0, rows, j0, j1, ks;
        tc_item(P, blockIdx.x, nst, m0, e, row0, rows, j0, j1, ks);
        int lvl;
        const int box = item_box(P, rows, &lvl);
        const uint32_t tx = (uint32_t)(ksub * (kABytes + box * kBK * 2));
        const CUtensorMap* am = &ta0;
        int am0 = m0;
        if (m0 >= g.seg2) { am = &ta2; am0 = m0 - g.seg2; }
        else if (m0 >= g.seg1) { am = &ta1; am0 = m0 - g.seg1; }
        pre = min(P.stages, j1 - j0);
        for (int i = 0; i < pre; ++i) {
          mbar_expect_tx(&full[i], tx);
          tma_load_3d(stage0 + (size_t)i * P.stage_bytes, am, &full[i], 0, am0, (j0 + i) * ksub);
        }
      }
      pdl_wait();
    }
    uint32_t kiter = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      int m0, e, row0, rows, j0, j1, ks;
      tc_item(P, item, nst, m0, e, row0, rows, j0, j1, ks);
      int lvl;
      const int box = item_box(P, rows, &lvl);
      const CUtensorMap* bm = box == g.ntile ? &tb : (lvl == 0 ? &tbs0 : lvl == 1 ? &tbs1 : &tbs2);
      const uint32_t tx = (uint32_t)(ksub * (n_a * kABytes + box * kBK * 2));
      const CUtensorMap* am = &ta0;
      int am0 = m0;
      if (g.mode == 0) {
        if (m0 >= g.seg2) { am = &ta2; am0 = m0 - g.seg2; }
        else if (m0 >= g.seg1) { am = &ta1; am0 = m0 - g.seg1; }
      }
      bool ok = true;
      for (int j = j0; j < j1; ++j, ++kiter) {
        const int s = kiter % P.stages;
        const uint32_t ph = (kiter / P.stages) & 1u;
        const int kb0 = j * ksub;
        uint8_t* st = stage0 + (size_t)s * P.stage_bytes;
        if (kiter < (uint32_t)pre) {   // weight box already in flight
          tma_load_3d(st + n_a * ksub * kABytes, bm, &full[s], 0, row0, kb0);
          continue;
        }
        if (!mbar_wait(&empty[s], ph ^ 1u, err, kErrTimeoutTma)) { ok = false; break; }
        mbar_expect_tx(&full[s], tx);
        if (g.mode == 0) {
          tma_load_3d(st, am, &full[s], 0, am0, kb0);
        } else {
          tma_load_4d(st, &ta0, &full[s], 0, m0, kb0, e);
          if (g.mode == 1) tma_load_4d(st + ksub * kABytes, &ta1, &full[s], 0, m0, kb0, e);
        }
        tma_load_3d(st + n_a * ksub * kABytes, bm, &full[s], 0, row0, kb0);
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t kiter = 0;
    int it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++it) {
      int m0, e, row0, rows, j0, j1, ks;
      tc_item(P, item, nst, m0, e, row0, rows, j0, j1, ks);
      const int n_mma = (rows + 15) & ~15;
      const uint32_t idesc = idesc_bf16(kBM, n_mma);
      int lvl;
      const int bsub = item_box(P, rows, &lvl) * kBK * 2;  // bytes of one token chunk in this item's box
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
        const int nsub = min(ksub, nk - j * ksub);
        const uint32_t st = smem_u32(stage0 + (size_t)s * P.stage_bytes);
        for (int u = 0; u < nsub; ++u) {
          const uint32_t sa = st + (uint32_t)(u * kABytes);
          const uint32_t sa1 = st + (uint32_t)((ksub + u) * kABytes);
          const uint32_t sb = st + (uint32_t)(n_a * ksub * kABytes + u * bsub);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = sdesc_k_sw128(sb + 32u * k);
            const uint32_t acc = (j > j0 || u > 0 || k > 0) ? 1u : 0u;
            umma_bf16(d0, sdesc_k_sw128(sa + 32u * k), bdesc, idesc, acc);
            if (n_a == 2) umma_bf16(d0 + (uint32_t)g.ntile, sdesc_k_sw128(sa1 + 32u * k), bdesc, idesc, acc);
          }
        }
        umma_commit(&empty[s]);
      }
      if (!ok) break;
      umma_commit(&acc_full[ab]);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // Per chunk of 32 token rows: each warp reads its 32-lane quarter of the
    // accumulator (row m = m0 + q*32 + lane, one column per token) and writes
    // it transposed into a [token][128] staging tile in shared memory; then
    // the 128 epilogue threads write whole output rows with 16-byte stores
    // (512 bytes of fp32, or 256 of bf16, per token row).  Writing the
    // accumulator column by column instead (one 128-byte store per warp
    // instruction) leaves the epilogue store-issue bound.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const int te = threadIdx.x - 64;  // 0..127 over the epilogue warps
    float* stg = reinterpret_cast<float*>(base + P.stages * P.stage_bytes + 1024);
    __nv_bfloat16* stg_b = reinterpret_cast<__nv_bfloat16*>(stg);
    const bool f32out = g.mode == 0 && (g.epi == EPI_STORE_F32 || g.epi == EPI_ADD_F32);
    float* out_f = reinterpret_cast<float*>(g.out);
    __nv_bfloat16* out_b = reinterpret_cast<__nv_bfloat16*>(g.out);
    // TMA-store form (dense fp32 stores): two staging tiles used in turn; the
    // thread that issues the stores (te 0) frees a tile by waiting for the
    // store issued from it two chunks earlier.
    const bool tstore = g.tma_out != 0;
    uint32_t chunk_no = 0;
    int it = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
      int m0, e, row0, rows, j0, j1, ks;
      tc_item(P, item, nst, m0, e, row0, rows, j0, j1, ks);
      const int ab = it % P.n_acc_buf;
      const uint32_t use = (uint32_t)(it / P.n_acc_buf);
      if (!mbar_wait(&acc_full[ab], use & 1u, err, kErrTimeoutEpi)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * P.acc_cols);
      const float bv = (g.bias && m0 + r < g.M) ? g.bias[m0 + r] : 0.f;
      const bool staged = (DG_EPI_STAGE_MODES >> g.mode) & 1;
      for (int c0 = 0; c0 < rows; c0 += kEpiRows) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
        if constexpr (kStats) {
          // sampler statistics instead of logits.  The chunk (32 tokens x 128
          // vocabulary rows) goes through the staging tile, XOR-swizzled so
          // that both the row-wise writes and the column-wise reads are free of
          // bank conflicts; then thread (warp q, lane t) reduces token t over
          // its 32-row group m0 + 32q .. +31 on its own, in vocabulary order.
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * kBM + (r ^ j)] = __uint_as_float(v[j]);
          named_barrier_sync(1, 128);
          const int t = lane, grp = (m0 >> 5) + q;
          float z[32];
          float mx = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int row = 32 * q + i;
            z[i] = m0 + row < g.M ? stg[t * kBM + (row ^ t)] * g.zscale : -INFINITY;
            mx = fmaxf(mx, z[i]);
          }
          named_barrier_sync(1, 128);   // the tile is rewritten by the next chunk
          VocabStat rec;
          rec.m = mx;
          rec.idx = m0 + 32 * q;
          rec.s = 0.f;
          rec.a = 0.f;
#pragma unroll
          for (int i = 31; i >= 0; --i)
            if (z[i] == mx) rec.idx = m0 + 32 * q + i;   // the first row holding the max
          if (g.argmax_mode) {
#pragma unroll
            for (int i = 0; i < 32; ++i) rec.s += z[i] == mx ? 1.f : 0.f;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float dz = z[i] - mx;
              const float e = expf(dz);                 // padding rows: exp(-inf) = 0
              rec.s += e;
              rec.a += e > 0.f ? e * dz : 0.f;
            }
          }
          if (c0 + t < rows && grp < g.n_groups)
            reinterpret_cast<VocabStat*>(g.out)[(size_t)(row0 + c0 + t) * g.n_groups + grp] = rec;
          continue;
        }
        if (!staged) {
          // direct form: each thread writes its row m, one token column at a time
          const int m = m0 + r;
          if (g.mode == 1) {
            uint32_t u[32];
            tmem_ld32(tbase + (uint32_t)(g.ntile + c0), u);
            tmem_ld_wait();
            if (m < g.M) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (c0 + j < rows) {
                  const float gt = __uint_as_float(v[j]), up = __uint_as_float(u[j]);
                  out_b[(size_t)(row0 + c0 + j) * g.ld_out + m] = __float2bfloat16_rn(swiglu_bf16(gt, up));
                }
              }
            }
          } else {
            tmem_ld_wait();
            if (m < g.M) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (c0 + j < rows) {
                  const float acc = __uint_as_float(v[j]) + bv;
                  const int tok = row0 + c0 + j;
                  if (g.mode == 2) out_b[(size_t)g.row_map[tok] * g.ld_out + m] = __float2bfloat16_rn(acc);
                  else if (g.epi == EPI_STORE_F32) out_f[(size_t)ks * g.split_stride + (size_t)tok * g.ld_out + m] = acc;
                  else if (g.epi == EPI_ADD_F32) out_f[(size_t)tok * g.ld_out + m] += acc;
                  else out_b[(size_t)tok * g.ld_out + m] = __float2bfloat16_rn(acc);
                }
              }
            }
          }
          continue;
        }
        if (g.mode == 1) {
          uint32_t u[32];
          tmem_ld32(tbase + (uint32_t)(g.ntile + c0), u);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gt = __uint_as_float(v[j]), up = __uint_as_float(u[j]);
            stg_b[j * kBM + r] = __float2bfloat16_rn(swiglu_bf16(gt, up));
          }
        } else if (tstore) {
          tmem_ld_wait();
          float* tile = stg + (chunk_no & 1u) * (kEpiBytes / 4);
          if (te == 0 && chunk_no >= 2) bulk_wait_read_1();
          named_barrier_sync(1, 128);  // the tile's previous store has finished reading it
#pragma unroll
          for (int j = 0; j < 32; ++j) tile[j * kBM + r] = __uint_as_float(v[j]) + bv;
          fence_proxy_async_smem();
          named_barrier_sync(1, 128);
          if (te == 0) {
            tma_store_3d(&tout, tile, m0, row0 + c0, ks);
            bulk_commit();
          }
          ++chunk_no;
          continue;
        } else if (f32out) {
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * kBM + r] = __uint_as_float(v[j]) + bv;
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) stg_b[j * kBM + r] = __float2bfloat16_rn(__uint_as_float(v[j]) + bv);
        }
        named_barrier_sync(1, 128);
        const int nrow = min(kEpiRows, rows - c0);
        if (f32out) {
#pragma unroll 4
          for (int it2 = 0; it2 < kEpiRows * 32 / 128; ++it2) {
            const int idx = it2 * 128 + te, row = idx >> 5, c4 = idx & 31;
            const int mm = m0 + c4 * 4;
            if (row < nrow && mm < g.M) {
              const int tok = row0 + c0 + row;
              float* dst = out_f + (size_t)ks * g.split_stride + (size_t)tok * g.ld_out + mm;
              const float4 val = *reinterpret_cast<const float4*>(stg + row * kBM + c4 * 4);
              const bool add = g.mode == 0 && g.epi == EPI_ADD_F32;
              if (P.vec && mm + 3 < g.M) {
                float4* d4 = reinterpret_cast<float4*>(dst);
                if (add) {
                  float4 o = *d4;
                  o.x += val.x; o.y += val.y; o.z += val.z; o.w += val.w;
                  *d4 = o;
                } else {
                  *d4 = val;
                }
              } else {
                const float vv[4] = {val.x, val.y, val.z, val.w};
                for (int c = 0; c < 4 && mm + c < g.M; ++c) dst[c] = add ? dst[c] + vv[c] : vv[c];
              }
            }
          }
        } else {
#pragma unroll 4
          for (int it2 = 0; it2 < kEpiRows * 16 / 128; ++it2) {
            const int idx = it2 * 128 + te, row = idx >> 4, c8 = idx & 15;
            const int mm = m0 + c8 * 8;
            if (row < nrow && mm < g.M) {
              const int tok = row0 + c0 + row;
              __nv_bfloat16* dst = out_b + (size_t)(g.mode == 2 ? g.row_map[tok] : tok) * g.ld_out + mm;
              const __nv_bfloat16* src = stg_b + row * kBM + c8 * 8;
              if (P.vec && mm + 7 < g.M) {
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
              } else {
                for (int c = 0; c < 8 && mm + c < g.M; ++c) dst[c] = src[c];
              }
            }
          }
        }
        named_barrier_sync(1, 128);  // the staging tile is reused by the next chunk
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
    if (tstore && te == 0) bulk_wait_read_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)P.tmem_cols);
  }
}

static void set_smem_attr() {
  static bool done = false;
  if (!done) {
    cudaFuncSetAttribute(gemm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    cudaFuncSetAttribute(gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    done = true;
  }
}

int launch_gemm_tc(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b,
                   const CUtensorMap* bsub, const TcGemm& g_in, int num_sms, cudaStream_t s, const CUtensorMap* tout) {
  TcGemm g = g_in;
  g.tma_out = (tout != nullptr && g.mode == 0 && g.epi == EPI_STORE_F32 && ((DG_EPI_STAGE_MODES & 1) != 0)) ? 1 : 0;
  const TcLayout L = tc_layout(g);
  if (L.stages < 2) return -1;   // the tile does not fit a two-stage pipeline
  TcKParams P;
  P.g = g;
  P.stages = L.stages;
  P.ksub = L.ksub;
  P.stage_bytes = L.stage_bytes;
  P.acc_cols = L.acc_cols;
  P.n_acc_buf = L.n_acc_buf;
  P.tmem_cols = L.tmem_cols;
  P.n_mtiles = (g.M + kBM - 1) / kBM;
  P.n_ttiles = (g.mode == 0) ? (g.T + g.ntile - 1) / g.ntile : 0;
  P.box_levels = 0;
  if (g.mode != 0 && bsub)
    while (P.box_levels < 3 && (32 << P.box_levels) < g.ntile) ++P.box_levels;
  {
    // 16-byte output vectors need aligned rows (and slices) in elements of the output type
    const bool f32out = g.mode == 0 && (g.epi == EPI_STORE_F32 || g.epi == EPI_ADD_F32);
    const int per_vec = f32out ? 4 : 8;
    P.vec = ((uintptr_t)g.out % 16 == 0) && g.ld_out % per_vec == 0 &&
            (g.ksplit <= 1 || g.split_stride % (size_t)per_vec == 0);
  }
  const int total = (g.mode == 0) ? P.n_mtiles * P.n_ttiles * (g.ksplit > 1 ? g.ksplit : 1)
                                  : g.n_work_max * P.n_mtiles;
  if (total <= 0) return 0;
  set_smem_attr();
  const int grid = std::min(total, num_sms * L.per_sm);
  const CUtensorMap& s0 = P.box_levels > 0 ? bsub[0] : b;
  const CUtensorMap& s1 = P.box_levels > 1 ? bsub[1] : b;
  const CUtensorMap& s2 = P.box_levels > 2 ? bsub[2] : b;
  launch_k(g.epi == EPI_VOCAB_STATS ? gemm_tc_kernel<true> : gemm_tc_kernel<false>, dim3(grid), dim3(kTcThreads), L.smem_bytes, s, a0, a1, a2, b, s0, s1, s2,
           g.tma_out ? *tout : b, P);
  return 0;
}

}  // namespace dg
