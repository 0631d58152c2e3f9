// tcgen05 attention on CTA pairs for the bf16 model with head dim 256 and an
// even number of query heads per KV head: the canvas step (every canvas query
// sees the whole cache and the whole canvas, [P1 二], [P2 架构基础]) and the
// causal encode of prompts / finished blocks.
//
// One pair (a cluster of two CTAs on neighbouring SMs) = (request b, query
// heads 2y and 2y+1, which read the same KV head g, 128-query tile, KV split).
// CTA r holds head 2y+r's 128 x 256 Q tile; the pair's MMAs run with M = 256
// (both heads' queries) and 128-key tiles:
//   S_j = Q K_j^T    M 256, N 128 keys, K 256: CTA r holds keys [64r, 64r+64)
//                    of the tile (64 x 256, 32 KB), so each K byte is loaded
//                    once for both heads;
//   O += P_j V_j     M 256, N 256 dims, K 128 keys: P_j from each CTA's TMEM,
//                    CTA r holds dims [128r, 128r+128) of V_j^T (32 KB).
// Each SM thus streams 64 KB of K/V per 128 keys for its 128 queries (a single
// CTA per head streams 128 KB), and each S instruction is 128 keys wide
// instead of 64.  Per CTA:
//   warp 0 lane 0: Q once, then the K halves (TMA, completing on the leader's
//     barriers, each CTA into its own shared memory);
//   warp 10 lane 0: the V^T halves;
//   warp 1 lane 0 of the leader: the MMA issuer; S_{j+2} goes out right behind
//     PV_j into the score buffer PV_j has just read (two buffers of 128 TMEM
//     columns; O holds the other 256), and every commit arrives on the barrier
//     of both CTAs;
//   warps 2-9: softmax over the CTA's own 128 rows, two threads per row (64
//     keys each): scores in log2 units, the running max raised only when a
//     tile exceeds it by more than 8 (then O and the running sum are rescaled
//     through TMEM), P (bf16) written back into TMEM over its own scores as the
//     A operand of PV.  Each softmax warp of both CTAs arrives once on the
//     leader's P barrier.  At the end O / l goes out as bf16, or O, max and sum to the
//     split workspace for the combine kernel.
// Every wait is bounded; both CTAs reach the final cluster barrier before the
// pair's TMEM is released.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "dg_pair.cuh"
#include "kernels.h"

namespace dg {

namespace {

constexpr int kA2Threads = 352;   // K producer, MMA issuer, 8 softmax warps, V producer
constexpr int kA2KStages = 3;     // K halves in flight (freed when their S MMA completes)
constexpr int kA2VStages = 2;     // V halves in flight (freed when their PV MMA completes)
constexpr int kA2QTile = 128;
constexpr int kA2KTile = 128;     // keys per tile (each CTA loads half of them)
constexpr int kA2Hd = 256;
constexpr int kA2QBytes = kA2QTile * kA2Hd * 2;               // 64 KB
constexpr int kA2KBytes = (kA2KTile / 2) * kA2Hd * 2;         // 32 KB: 64 keys x 256 dims
constexpr int kA2VBox = (kA2Hd / 2) * 64 * 2;                 // 16 KB: 128 dims x 64 keys
constexpr int kA2VBytes = 2 * kA2VBox;                        // 32 KB: 128 dims x 128 keys
constexpr int kA2RedBytes = 256 * 4;
constexpr int kA2BarBytes = 192;
constexpr int kA2Smem =
    1008 + kA2QBytes + kA2KStages * kA2KBytes + kA2VStages * kA2VBytes + kA2RedBytes + kA2BarBytes;
static_assert((1 + 2 * kA2KStages + 2 * kA2VStages + 3 * 2) * 8 + 4 <= kA2BarBytes, "barrier area");
static_assert(kA2Smem <= 232448, "shared memory");
constexpr float kA2RescaleThreshold = 8.0f;   // log2 units

struct Attn2Params {
  AttnTcArgs t;
  int n_qtiles;
  float scale_log2;   // log2(e) / sqrt(hd)
  int has_tpo;        // split partials go out through TMA stores (tpo valid)
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kA2Threads, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tpo,
                    __nv_bfloat16* __restrict__ out, const Attn2Params P) {
  extern __shared__ uint8_t smem_raw[];
  const AttnArgs& a = P.t.a;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int split = pair % P.t.n_split;
  const int qt = pair / P.t.n_split;
  const int h = 2 * blockIdx.y + (int)rank, b = blockIdx.z;
  const int g = h * a.hkv / a.hq;          // the same for both heads of the pair
  const int slot = a.bi.slot[b], plen = a.bi.len[b];
  const int q0 = qt * kA2QTile;
  const int n_keys = plen + a.nq;
  const int kmax = a.causal ? min(n_keys, plen + q0 + kA2QTile) : n_keys;
  const int tiles_all = (kmax + kA2KTile - 1) / kA2KTile;
  const int per = (tiles_all + P.t.n_split - 1) / P.t.n_split;
  const int t_begin = split * per;
  const int t_end = min(tiles_all, t_begin + per);
  const int ntiles = max(0, t_end - t_begin);   // the same for both CTAs of the pair
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_id = ((size_t)b * a.hq + h) * a.nq;   // first output row of this (b, h)

  if (ntiles == 0) {
    // empty split (causal tail): contributes nothing to the combine.  Both
    // CTAs of the pair leave here, before any cluster-wide step.
    pdl_wait();
    pdl_trigger();
    if (warp >= 2 && warp < 6) {
      const int r = (warp & 3) * 32 + lane;
      const int qi = q0 + r;
      if (qi < a.nq && P.t.n_split > 1) {
        const size_t pr = (size_t)split * a.B * a.hq * a.nq + row_id + qi;
        P.t.part_ml[2 * pr] = -INFINITY;
        P.t.part_ml[2 * pr + 1] = 0.f;
        float* po = P.t.part_o + pr * kA2Hd;
        for (int d = 0; d < kA2Hd; ++d) po[d] = 0.f;
      }
    }
    return;
  }

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kA2QBytes;                   // [kA2KStages][kA2KBytes]
  uint8_t* sV = sK + kA2KStages * kA2KBytes;      // [kA2VStages][kA2VBytes]
  float* red = reinterpret_cast<float*>(sV + kA2VStages * kA2VBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kA2VStages * kA2VBytes + kA2RedBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;             // [kA2KStages]  leader: both K halves landed
  uint64_t* k_empty = k_full + kA2KStages;   // [kA2KStages]  both: S MMA done with the stage
  uint64_t* v_full = k_empty + kA2KStages;   // [kA2VStages]  leader: both V halves landed
  uint64_t* v_empty = v_full + kA2VStages;   // [kA2VStages]  both: PV MMA done with the stage
  uint64_t* s_full = v_empty + kA2VStages;   // [2]           both: S in TMEM
  uint64_t* p_full = s_full + 2;             // [2]           leader: both CTAs' P in TMEM
  uint64_t* pv_done = p_full + 2;            // [2]           both: PV done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 2);
  int* err = P.t.err;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kA2KStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kA2VStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 2 * 8);   // one arrival per softmax warp of either CTA
      mbar_init(&pv_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc2(tmem_slot, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touches no global memory: it overlaps the previous kernel
  pdl_wait();
  pdl_trigger();
  const uint32_t tS = tmem;          // score buffers: columns [128 s, 128 s + 128), s < 2
  const uint32_t tO = tmem + 256;    // output accumulator: columns [256, 512)

  if (warp == 0 && lane == 0) {
    // ----------------------------------------------------------- Q and K
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    const int qrow = (int)row_id + q0;
    if (leader) mbar_expect_tx(q_full, 2 * kA2QBytes);
    tma_load_3d_pair(sQ, &tq, map_to_rank(q_full, 0), 0, qrow, 0);
    const int krow = (slot * a.hkv + g) * a.max_ctx + (int)rank * (kA2KTile / 2);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kA2KStages;
      const uint32_t ph = (uint32_t)(j / kA2KStages) & 1u;
      if (!mbar_wait(&k_empty[s], ph ^ 1u, err, kErrTimeoutAttn)) break;
      if (leader) mbar_expect_tx(&k_full[s], 2 * kA2KBytes);
      tma_load_3d_pair(sK + s * kA2KBytes, &tk, map_to_rank(&k_full[s], 0), 0, krow + (t_begin + j) * kA2KTile, 0);
    }
  } else if (warp == 10 && lane == 0) {
    // ----------------------------------------------------------- V^T
    prefetch_tmap(&tv);
    const int vrow = (slot * a.hkv + g) * kA2Hd + (int)rank * (kA2Hd / 2);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kA2VStages;
      const uint32_t ph = (uint32_t)(j / kA2VStages) & 1u;
      if (!mbar_wait(&v_empty[s], ph ^ 1u, err, kErrTimeoutAttn)) break;
      if (leader) mbar_expect_tx(&v_full[s], 2 * kA2VBytes);
      const uint32_t vb = map_to_rank(&v_full[s], 0);
      const int key0 = (t_begin + j) * kA2KTile;
      tma_load_2d_pair(sV + s * kA2VBytes, &tv, vb, key0, vrow);
      tma_load_2d_pair(sV + s * kA2VBytes + kA2VBox, &tv, vb, key0 + 64, vrow);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ----------------------------------------------------------- MMA issuer
    const uint32_t idesc_s = idesc_bf16(2 * kA2QTile, kA2KTile);
    const uint32_t idesc_o = idesc_bf16(2 * kA2QTile, kA2Hd);
    const uint32_t q_base = smem_u32(sQ);
    bool ok = mbar_wait(q_full, 0, err, kErrTimeoutAttn);
    auto issue_s = [&](int j) -> bool {
      const int s = j & 1;
      const int ks = j % kA2KStages;
      // S_j reuses the TMEM columns of P_{j-2}; PV_{j-2} was issued earlier,
      // and the tcgen05.mma of one thread run in issue order.
      if (!mbar_wait(&k_full[ks], (uint32_t)(j / kA2KStages) & 1u, err, kErrTimeoutAttn)) return false;
      tc_fence_after();
      const uint32_t k_base = smem_u32(sK + ks * kA2KBytes);
#pragma unroll
      for (int c = 0; c < kA2Hd / 64; ++c)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma2_bf16(tS + (uint32_t)(s * kA2KTile), sdesc_k_sw128(q_base + c * (kA2QTile * 128) + 32u * k),
                     sdesc_k_sw128(k_base + c * ((kA2KTile / 2) * 128) + 32u * k), idesc_s, (c | k) ? 1u : 0u);
      umma2_commit_both(&s_full[s]);
      umma2_commit_both(&k_empty[ks]);
      return true;
    };
    for (int j = 0; j < min(ntiles, 2) && ok; ++j) ok = issue_s(j);
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j & 1;
      const int vs = j % kA2VStages;
      if (!mbar_wait(&p_full[s], (uint32_t)(j >> 1) & 1u, err, kErrTimeoutAttn)) break;
      if (!mbar_wait(&v_full[vs], (uint32_t)(j / kA2VStages) & 1u, err, kErrTimeoutAttn)) break;
      tc_fence_after();
      // O += P_j V_j: P_j (bf16, 64 columns) read from TMEM where S_j was;
      // 16 keys per instruction, 64 keys per V^T box
      const uint32_t v_base = smem_u32(sV + vs * kA2VBytes);
#pragma unroll
      for (int i = 0; i < kA2KTile / 16; ++i)
        umma2_bf16_ts(tO, tS + (uint32_t)(s * kA2KTile + 8 * i),
                      sdesc_k_sw128(v_base + (uint32_t)((i >> 2) * kA2VBox) + 32u * (i & 3)), idesc_o,
                      (j > 0 || i > 0) ? 1u : 0u);
      umma2_commit_both(&pv_done[s]);
      umma2_commit_both(&v_empty[vs]);
      if (j + 2 < ntiles && !issue_s(j + 2)) break;
    }
  } else if (warp >= 2 && warp < 10) {
    // ----------------------------------------------------------- softmax
    // 8 warps: thread (quarter, lane) of half hf owns query row r and keys
    // [64 hf, 64 hf + 64) of each 128-key tile, and O columns [128 hf, +128).
    // The two halves of a row agree on the tile max through shared memory.
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int row_lim = a.causal ? min(n_keys, plen + qi + 1) : n_keys;  // keys < row_lim are visible
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j & 1;
      const uint32_t ph = (uint32_t)(j >> 1) & 1u;
      if (!mbar_wait(&s_full[s], ph, err, kErrTimeoutAttn)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tcol = tS + lane_off + (uint32_t)(s * kA2KTile + hf * 64);
      float x[64];
      {
        uint32_t sv[32];
        tmem_ld32(tcol, sv);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(sv[c]);
        tmem_ld32(tcol + 32u, sv);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[32 + c] = __uint_as_float(sv[c]);
      }
      // x stays in raw score units (the log2 scale is folded into the
      // exponent below); the max runs as four independent chains
      const int kbase = (t_begin + j) * kA2KTile + hf * 64;
      if (kbase + 64 > row_lim) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = (kbase + c < row_lim) ? x[c] : -INFINITY;
      }
      float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int c = 4; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], x[c]);
      const float hmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * P.scale_log2;
      // tile max of the row: exchange with the other half.  The barrier also
      // orders both halves' reads of S before any P write into these columns.
      red[hf * 128 + r] = hmax;
      named_barrier_sync(1, 256);
      const float tmax = fmaxf(hmax, red[(hf ^ 1) * 128 + r]);
      named_barrier_sync(1, 256);   // both halves have read before the buffer is reused
      // raise the running max only when this tile exceeds it by the threshold
      const bool raise = tmax > m_run + kA2RescaleThreshold;
      const float m_new = raise ? tmax : m_run;
      const float alpha = (raise && m_run > -INFINITY) ? fast_exp2(m_run - m_new) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f) && j > 0) {
        // O of rows in this warp must be rescaled: wait until PV_{j-1} landed
        if (!mbar_wait(&pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, err, kErrTimeoutAttn)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kA2Hd / 2; c0 += 32) {
          uint32_t ov[32];
          const uint32_t ta = tO + lane_off + (uint32_t)(hf * (kA2Hd / 2) + c0);
          tmem_ld32(ta, ov);
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(ta, ov);
        }
        tmem_st_wait();
      }
      l_run *= alpha;
      m_run = m_new;
      // P_j (bf16) overwrites the first 64 columns of S_j's TMEM buffer:
      // half hf's 64 keys are 32 packed columns at 32 hf.
      // (x[e] is reused for the pair sums: x[2e], x[2e+1] are read before x[e] is written)
      uint32_t pk[32];
      const bool live = m_run > -INFINITY;
      const float sc = P.scale_log2, nm = -m_run;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = live ? fast_exp2(fmaf(x[2 * e], sc, nm)) : 0.f;
        const float p1 = live ? fast_exp2(fmaf(x[2 * e + 1], sc, nm)) : 0.f;
        const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
        pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
        x[e] = __low2float(pp) + __high2float(pp);   // sum what the MMA will see
      }
      tmem_st32(tS + lane_off + (uint32_t)(s * kA2KTile + hf * 32), pk);
#pragma unroll
      for (int w2 = 16; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int e = 0; e < w2; ++e) x[e] += x[e + w2];
      l_run += x[0];
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(&p_full[s], 0));
    }
    // the row sum is the sum of both halves
    if (ok) {
      red[hf * 128 + r] = l_run;
      named_barrier_sync(1, 256);
      l_run += red[(hf ^ 1) * 128 + r];
    }
    if (ok) ok = mbar_wait(&pv_done[(ntiles - 1) & 1], (uint32_t)((ntiles - 1) >> 1) & 1u, err, kErrTimeoutAttn);
    if (ok) {
      tc_fence_after();
      const bool valid = qi < a.nq;
      const int cbase = hf * (kA2Hd / 2);
      if (P.t.n_split == 1) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* op = out + ((size_t)b * a.nq + qi) * ((size_t)a.hq * kA2Hd) + (size_t)h * kA2Hd + cbase;
#pragma unroll 1
        for (int c0 = 0; c0 < kA2Hd / 2; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + lane_off + (uint32_t)(cbase + c0), ov);
          if (valid) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint32_t pq[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 pp = __floats2bfloat162_rn(__uint_as_float(ov[c + 2 * e]) * inv,
                                                                __uint_as_float(ov[c + 2 * e + 1]) * inv);
                pq[e] = *reinterpret_cast<const uint32_t*>(&pp);
              }
              *reinterpret_cast<uint4*>(op + c0 + c) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
            }
          }
        }
      } else if (P.has_tpo) {
        // Partial O through the (now idle) K/V stages: 8 tiles of 128 rows x
        // 32 columns (fp32, 128-byte swizzle: 16-byte chunk k of row r at
        // chunk k ^ (r & 7)), then 8 TMA stores; rows past nq are clipped.
        const size_t pr = (size_t)split * a.B * a.hq * a.nq + row_id + qi;
        if (valid && hf == 0) {
          P.t.part_ml[2 * pr] = m_run;
          P.t.part_ml[2 * pr + 1] = l_run;
        }
        float* stage = reinterpret_cast<float*>(sK);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tO + lane_off + (uint32_t)(cbase + 32 * cc), ov);
          float* row = stage + (hf * 4 + cc) * (kA2QTile * 32) + r * 32;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(row + 4 * (k ^ (r & 7))) =
                make_float4(__uint_as_float(ov[4 * k]), __uint_as_float(ov[4 * k + 1]),
                            __uint_as_float(ov[4 * k + 2]), __uint_as_float(ov[4 * k + 3]));
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, 256);
        if (warp == 2 && lane == 0) {
          const int plane = (split * a.B + b) * a.hq + h;
          for (int t2 = 0; t2 < 8; ++t2)
            tma_store_3d(&tpo, stage + t2 * (kA2QTile * 32), (t2 >> 2) * (kA2Hd / 2) + 32 * (t2 & 3), q0, plane);
          bulk_commit();
          bulk_wait_read_all();
        }
      } else {
        const size_t pr = (size_t)split * a.B * a.hq * a.nq + row_id + qi;
        if (valid && hf == 0) {
          P.t.part_ml[2 * pr] = m_run;
          P.t.part_ml[2 * pr + 1] = l_run;
        }
        float* po = P.t.part_o + pr * kA2Hd + cbase;
#pragma unroll 1
        for (int c0 = 0; c0 < kA2Hd / 2; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tO + lane_off + (uint32_t)(cbase + c0), ov);
          if (valid) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(po + c0 + c) =
                  make_float4(__uint_as_float(ov[c]), __uint_as_float(ov[c + 1]), __uint_as_float(ov[c + 2]),
                              __uint_as_float(ov[c + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();     // the leader's last MMAs have read both CTAs' tiles; TMEM is idle
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

}  // namespace

bool attn_tc2_supported(int hq, int hkv, int hd) { return hd == kA2Hd && hkv > 0 && hq % (2 * hkv) == 0; }

void launch_attn_tc2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap* tpo,
                     __nv_bfloat16* out, const AttnTcArgs& t, cudaStream_t s) {
  const AttnArgs& a = t.a;
  if (a.B <= 0 || a.nq <= 0) return;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(attn_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kA2Smem);
    attr = true;
  }
  Attn2Params P;
  P.t = t;
  P.n_qtiles = (a.nq + kA2QTile - 1) / kA2QTile;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)a.hd);
  P.has_tpo = (t.n_split > 1 && tpo) ? 1 : 0;
  dim3 grid(2 * P.n_qtiles * t.n_split, a.hq / 2, a.B);
  launch_k(attn_tc2_kernel, dim3(grid), dim3(kA2Threads), kA2Smem, s, tq, tk, tv, P.has_tpo ? *tpo : tv, out, P);
  if (t.n_split > 1) launch_attn_combine(t.part_o, t.part_ml, out, t.n_split, a.B, a.hq, a.nq, s);
}

}  // namespace dg
