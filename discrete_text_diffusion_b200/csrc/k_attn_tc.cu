// tcgen05 attention for the bf16 model with head dim 256: the canvas step
// (every canvas query sees the whole cache and the whole canvas, [P1 二],
// [P2 架构基础]) and the causal encode of prompts / finished blocks.
//
// One CTA = (request b, query head h, 128-query tile, KV split).  GQA: head h
// reads KV head h*Hkv/Hq.
//   warp 0 lane 0: TMA producer.  Q tile (128 x 256) once; then per 64-key tile
//     the K tile (64 keys x 256) and the transposed V tile (256 x 64 keys)
//     into one of two stages.
//   warp 1 lane 0: MMA issuer.  S_j = Q K_j^T (M 128, N 64, K 256) into one of
//     kSBuf TMEM score buffers, queued kSBuf tiles ahead: S_{j+kSBuf} right
//     behind O += P_j V_j (M 128, N 256, K 64), O resident in TMEM (256
//     columns).  Per-tile timers show the tensor pipe busy ~1500 of ~2850
//     cycles: the 16 S instructions (N = 64, both operands in shared memory)
//     run at about half the rate of the 4 PV instructions.
//   warps 2-9: softmax, two threads per query row (32 keys each).  Scores
//     are scaled to log2 units; the running max is only raised when a tile
//     exceeds it by more than 8 (then O and the running sum are rescaled
//     through TMEM), so most tiles need no correction.  P (bf16) is written
//     back into TMEM over its own scores and is the A operand of the PV MMA,
//     so it never touches shared memory.  At the end O / l goes out as bf16,
//     or O, max and sum go to the split workspace for the combine kernel.
#include <cuda_bf16.h>

#include <algorithm>

#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

constexpr int kAttnThreads = 352;   // K producer, MMA issuer, 8 softmax warps, V producer
constexpr int kKStages = 3;         // K tiles in flight (freed when their S MMA completes)
constexpr int kVStages = 2;         // V tiles in flight (freed when their PV MMA completes)
constexpr int kQTile = 128;
constexpr int kKTile = 64;
constexpr int kHd = 256;
constexpr int kQBytes = kQTile * kHd * 2;   // 64 KB
constexpr int kKBytes = kKTile * kHd * 2;   // 32 KB
constexpr int kVBytes = kHd * kKTile * 2;   // 32 KB
constexpr int kSBuf = 2;                      // TMEM score buffers (64 columns each; O uses [256, 512)); 3 measured no faster
constexpr int kRedBytes = 256 * 4;           // per-row exchange between the two halves
constexpr int kBarBytes = 192;               // mbarriers and the TMEM slot
constexpr int kAttnSmem = 1008 + kQBytes + kKStages * kKBytes + kVStages * kVBytes + kRedBytes + kBarBytes;
static_assert((1 + 2 * kKStages + 2 * kVStages + 3 * kSBuf) * 8 + 4 <= kBarBytes, "barrier area");
static_assert(kSBuf * kKTile <= 256, "score buffers must stay below the O columns");
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct AttnTcParams {
  AttnTcArgs t;
  int n_qtiles;
  float scale_log2;   // log2(e) / sqrt(hd)
};

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, __nv_bfloat16* __restrict__ out, const AttnTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const AttnArgs& a = P.t.a;
  const int split = blockIdx.x % P.t.n_split;
  const int qt = blockIdx.x / P.t.n_split;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h * a.hkv / a.hq;
  const int slot = a.bi.slot[b], plen = a.bi.len[b];
  const int q0 = qt * kQTile;
  const int n_keys = plen + a.nq;
  const int kmax = a.causal ? min(n_keys, plen + q0 + kQTile) : n_keys;
  const int tiles_all = (kmax + kKTile - 1) / kKTile;
  const int per = (tiles_all + P.t.n_split - 1) / P.t.n_split;
  const int t_begin = split * per;
  const int t_end = min(tiles_all, t_begin + per);
  const int ntiles = max(0, t_end - t_begin);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_id = ((size_t)b * a.hq + h) * a.nq;   // first output row of this (b, h)

  if (ntiles == 0) {
    // empty split (causal tail): contributes nothing to the combine
    pdl_wait();
    pdl_trigger();
    if (warp >= 2 && warp < 6) {
      const int r = (warp & 3) * 32 + lane;
      const int qi = q0 + r;
      if (qi < a.nq && P.t.n_split > 1) {
        const size_t pr = (size_t)split * a.B * a.hq * a.nq + row_id + qi;
        P.t.part_ml[2 * pr] = -INFINITY;
        P.t.part_ml[2 * pr + 1] = 0.f;
        float* po = P.t.part_o + pr * kHd;
        for (int d = 0; d < kHd; ++d) po[d] = 0.f;
      }
    }
    return;
  }

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kQBytes;                  // [kKStages][kKBytes]
  uint8_t* sV = sK + kKStages * kKBytes;       // [kVStages][kVBytes]
  float* red = reinterpret_cast<float*>(sV + kVStages * kVBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVStages * kVBytes + kRedBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;          // [kKStages]
  uint64_t* k_empty = k_full + kKStages;  // [kKStages]
  uint64_t* v_full = k_empty + kKStages;  // [kVStages]
  uint64_t* v_empty = v_full + kVStages;  // [kVStages]
  uint64_t* s_full = v_empty + kVStages;  // [kSBuf]
  uint64_t* p_full = s_full + kSBuf;      // [kSBuf]
  uint64_t* pv_done = p_full + kSBuf;     // [kSBuf]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + kSBuf);
  int* err = P.t.err;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
      mbar_init(&pv_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touches no global memory: it overlaps the previous kernel
  pdl_wait();
  pdl_trigger();
  const uint32_t tS = tmem;          // score buffers: columns [64 s, 64 s + 64), s < kSBuf
  const uint32_t tO = tmem + 256;    // output accumulator: columns [256, 512)

  if (warp == 0 && lane == 0) {
    // ----------------------------------------------------------- K producer
    // One TMA instruction each for Q (4 chunks of 64 dims) and every K tile.
    // K and V have separate rings: a K tile is free as soon as its S MMA is
    // done, so the next K loads start a tile earlier than a shared ring allows.
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    const int qrow = (int)row_id + q0;
    mbar_expect_tx(q_full, kQBytes);
    tma_load_3d(sQ, &tq, q_full, 0, qrow, 0);
    const int krow = (slot * a.hkv + g) * a.max_ctx;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kKStages;
      const uint32_t ph = (uint32_t)(j / kKStages) & 1u;
      if (!mbar_wait(&k_empty[s], ph ^ 1u, err, kErrTimeoutAttn)) break;
      mbar_expect_tx(&k_full[s], kKBytes);
      tma_load_3d(sK + s * kKBytes, &tk, &k_full[s], 0, krow + (t_begin + j) * kKTile, 0);
    }
  } else if (warp == 10 && lane == 0) {
    // ----------------------------------------------------------- V producer
    prefetch_tmap(&tv);
    const int vrow = (slot * a.hkv + g) * kHd;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kVStages;
      const uint32_t ph = (uint32_t)(j / kVStages) & 1u;
      if (!mbar_wait(&v_empty[s], ph ^ 1u, err, kErrTimeoutAttn)) break;
      mbar_expect_tx(&v_full[s], kVBytes);
      tma_load_2d(sV + s * kVBytes, &tv, &v_full[s], (t_begin + j) * kKTile, vrow);
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- MMA issuer
    const uint32_t idesc_s = idesc_bf16(kQTile, kKTile);
    const uint32_t idesc_o = idesc_bf16(kQTile, kHd);
    const uint32_t q_base = smem_u32(sQ);
    bool ok = mbar_wait(q_full, 0, err, kErrTimeoutAttn);
    auto issue_s = [&](int j) -> bool {
      const int s = j % kSBuf;
      const int ks = j % kKStages;
      // S_j reuses the TMEM columns of P_{j-kSBuf}; PV_{j-kSBuf} was issued
      // earlier, and the tcgen05.mma of one thread run in issue order.
      if (!mbar_wait(&k_full[ks], (uint32_t)(j / kKStages) & 1u, err, kErrTimeoutAttn)) return false;
      tc_fence_after();
      const uint32_t k_base = smem_u32(sK + ks * kKBytes);
#pragma unroll
      for (int c = 0; c < kHd / 64; ++c)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tS + (uint32_t)(s * kKTile), sdesc_k_sw128(q_base + c * (kQTile * 128) + 32u * k),
                    sdesc_k_sw128(k_base + c * (kKTile * 128) + 32u * k), idesc_s, (c | k) ? 1u : 0u);
      umma_commit(&s_full[s]);
      umma_commit(&k_empty[ks]);
      return true;
    };
    for (int j = 0; j < min(ntiles, kSBuf) && ok; ++j) ok = issue_s(j);
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j % kSBuf;
      const int vs = j % kVStages;
      if (!mbar_wait(&p_full[s], (uint32_t)(j / kSBuf) & 1u, err, kErrTimeoutAttn)) break;
      if (!mbar_wait(&v_full[vs], (uint32_t)(j / kVStages) & 1u, err, kErrTimeoutAttn)) break;
      tc_fence_after();
      // O += P_j V_j with P_j (bf16, 32 columns) read from TMEM where S_j was
      const uint32_t v_base = smem_u32(sV + vs * kVBytes);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_bf16_ts(tO, tS + (uint32_t)(s * kKTile + 8 * k), sdesc_k_sw128(v_base + 32u * k), idesc_o,
                     (j > 0 || k > 0) ? 1u : 0u);
      umma_commit(&pv_done[s]);
      umma_commit(&v_empty[vs]);
      if (j + kSBuf < ntiles && !issue_s(j + kSBuf)) break;
    }
  } else if (warp >= 2 && warp < 10) {
    // ----------------------------------------------------------- softmax
    // 8 warps: thread (quarter, lane) of half hf owns query row r and keys
    // [32 hf, 32 hf + 32) of each 64-key tile, and O columns [128 hf, +128).
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
      const int s = j % kSBuf;
      const uint32_t ph = (uint32_t)(j / kSBuf) & 1u;
      if (!mbar_wait(&s_full[s], ph, err, kErrTimeoutAttn)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(tS + lane_off + (uint32_t)(s * kKTile + hf * 32), sv);
      const int kbase = (t_begin + j) * kKTile + hf * 32;
      float x[32];
      float hmax = -INFINITY;
      if (kbase + 32 <= row_lim) {
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[c] = __uint_as_float(sv[c]) * P.scale_log2; hmax = fmaxf(hmax, x[c]); }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = (kbase + c < row_lim) ? __uint_as_float(sv[c]) * P.scale_log2 : -INFINITY;
          hmax = fmaxf(hmax, x[c]);
        }
      }
      // tile max of the row: exchange with the other half.  The barrier also
      // orders both halves' reads of S before any P write into these columns.
      red[hf * 128 + r] = hmax;
      named_barrier_sync(1, 256);
      const float tmax = fmaxf(hmax, red[(hf ^ 1) * 128 + r]);
      named_barrier_sync(1, 256);   // both halves have read before the buffer is reused
      // raise the running max only when this tile exceeds it by the threshold
      const bool raise = tmax > m_run + kRescaleThreshold;
      const float m_new = raise ? tmax : m_run;
      const float alpha = (raise && m_run > -INFINITY) ? fast_exp2(m_run - m_new) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f) && j > 0) {
        // O of rows in this warp must be rescaled: wait until PV_{j-1} landed
        if (!mbar_wait(&pv_done[(j - 1) % kSBuf], (uint32_t)((j - 1) / kSBuf) & 1u, err, kErrTimeoutAttn)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kHd / 2; c0 += 32) {
          uint32_t ov[32];
          const uint32_t ta = tO + lane_off + (uint32_t)(hf * (kHd / 2) + c0);
          tmem_ld32(ta, ov);
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(ta, ov);
        }
        tmem_st_wait();
      }
      l_run *= alpha;
      m_run = m_new;
      // P_j (bf16) overwrites the first 32 columns of S_j's TMEM buffer:
      // half hf's 32 keys are 16 packed columns at 16 hf.
      uint32_t pk[16];
      float ps[16];
      const bool live = m_run > -INFINITY;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float p0 = live ? fast_exp2(x[2 * e] - m_run) : 0.f;
        const float p1 = live ? fast_exp2(x[2 * e + 1] - m_run) : 0.f;
        const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
        pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
        ps[e] = __low2float(pp) + __high2float(pp);   // sum what the MMA will see
      }
      tmem_st16_wait(tS + lane_off + (uint32_t)(s * kKTile + hf * 16), pk);
#pragma unroll
      for (int w2 = 8; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int e = 0; e < w2; ++e) ps[e] += ps[e + w2];
      l_run += ps[0];
      tc_fence_before();
      mbar_arrive(&p_full[s]);
    }
    // the row sum is the sum of both halves
    if (ok) {
      red[hf * 128 + r] = l_run;
      named_barrier_sync(1, 256);
      l_run += red[(hf ^ 1) * 128 + r];
    }
    if (ok)
      ok = mbar_wait(&pv_done[(ntiles - 1) % kSBuf], (uint32_t)((ntiles - 1) / kSBuf) & 1u, err, kErrTimeoutAttn);
    if (ok) {
      tc_fence_after();
      const bool valid = qi < a.nq;
      const int cbase = hf * (kHd / 2);
      if (P.t.n_split == 1) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* op = out + ((size_t)b * a.nq + qi) * ((size_t)a.hq * kHd) + (size_t)h * kHd + cbase;
#pragma unroll 1
        for (int c0 = 0; c0 < kHd / 2; c0 += 32) {
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
      } else {
        const size_t pr = (size_t)split * a.B * a.hq * a.nq + row_id + qi;
        if (valid && hf == 0) {
          P.t.part_ml[2 * pr] = m_run;
          P.t.part_ml[2 * pr + 1] = l_run;
        }
        float* po = P.t.part_o + pr * kHd + cbase;
#pragma unroll 1
        for (int c0 = 0; c0 < kHd / 2; c0 += 32) {
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
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the split partials of one (b, h, query) row: one warp per row, lane
// l owning columns [8l, 8l + 8) (two 16-byte loads per split, one 16-byte
// store).  The loads of all splits are independent and issued together.  A
// split that saw no key (max -inf) contributes nothing, whatever its O holds.
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                    __nv_bfloat16* __restrict__ out, int n_split, int B, int hq, int nq) {
  pdl_wait();
  pdl_trigger();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = B * hq * nq;
  if (row >= rows) return;
  const size_t stride = (size_t)rows;
  float M = -INFINITY;
  float L = 0.f;
  float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
  if (n_split <= 8) {
    // every split's (max, sum) and O columns in flight at once: one memory latency per row
    float2 ml[8];
    float4 v0[8], v1[8];
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < n_split) {
        ml[s] = *reinterpret_cast<const float2*>(part_ml + 2 * (s * stride + row));
        const float4* po = reinterpret_cast<const float4*>(part_o + (s * stride + row) * kHd) + 2 * lane;
        v0[s] = po[0];
        v1[s] = po[1];
      }
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < n_split) M = fmaxf(M, ml[s].x);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < n_split && ml[s].x != -INFINITY) {
        const float w = exp2f(ml[s].x - M);
        L += ml[s].y * w;
        a0.x += w * v0[s].x; a0.y += w * v0[s].y; a0.z += w * v0[s].z; a0.w += w * v0[s].w;
        a1.x += w * v1[s].x; a1.y += w * v1[s].y; a1.z += w * v1[s].z; a1.w += w * v1[s].w;
      }
  } else {
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, part_ml[2 * (s * stride + row)]);
#pragma unroll 4
    for (int s = 0; s < n_split; ++s) {
      const float ms = part_ml[2 * (s * stride + row)];
      const float ls = part_ml[2 * (s * stride + row) + 1];
      const float4* po = reinterpret_cast<const float4*>(part_o + (s * stride + row) * kHd) + 2 * lane;
      const float4 v0 = po[0], v1 = po[1];
      const bool live = ms != -INFINITY;
      const float w = live ? exp2f(ms - M) : 0.f;
      if (live) {
        L += ls * w;
        a0.x += w * v0.x; a0.y += w * v0.y; a0.z += w * v0.z; a0.w += w * v0.w;
        a1.x += w * v1.x; a1.y += w * v1.y; a1.z += w * v1.z; a1.w += w * v1.w;
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  // row = (b*hq + h)*nq + q  ->  out[(b*nq + q), h*hd + d]
  const int q = row % nq;
  const int bh = row / nq;
  const int h = bh % hq, b = bh / hq;
  __nv_bfloat16* op = out + ((size_t)b * nq + q) * ((size_t)hq * kHd) + (size_t)h * kHd + 8 * lane;
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(a0.x * inv, a0.y * inv), p1 = __floats2bfloat162_rn(a0.z * inv, a0.w * inv);
  const __nv_bfloat162 p2 = __floats2bfloat162_rn(a1.x * inv, a1.y * inv), p3 = __floats2bfloat162_rn(a1.z * inv, a1.w * inv);
  uint4 u;
  u.x = *reinterpret_cast<const uint32_t*>(&p0);
  u.y = *reinterpret_cast<const uint32_t*>(&p1);
  u.z = *reinterpret_cast<const uint32_t*>(&p2);
  u.w = *reinterpret_cast<const uint32_t*>(&p3);
  *reinterpret_cast<uint4*>(op) = u;
}

size_t attn_tc_partial_floats(int n_split, int B, int hq, int nq_pad, int hd) {
  return (size_t)n_split * B * hq * nq_pad * hd;
}

void launch_attn_combine(const float* part_o, const float* part_ml, __nv_bfloat16* out, int n_split, int B, int hq,
                         int nq, cudaStream_t s) {
  const int rows = B * hq * nq;
  if (rows <= 0) return;
  launch_k(attn_combine_kernel, dim3((rows * 32 + 255) / 256), dim3(256), 0, s, part_o, part_ml, out, n_split, B, hq,
           nq);
}

void launch_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, __nv_bfloat16* out,
                    const AttnTcArgs& t, cudaStream_t s) {
  const AttnArgs& a = t.a;
  if (a.B <= 0 || a.nq <= 0) return;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
    attr = true;
  }
  AttnTcParams P;
  P.t = t;
  P.n_qtiles = (a.nq + kQTile - 1) / kQTile;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)a.hd);
  dim3 grid(P.n_qtiles * t.n_split, a.hq, a.B);
  launch_k(attn_tc_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmem, s, tq, tk, tv, out, P);
  if (t.n_split > 1) launch_attn_combine(t.part_o, t.part_ml, out, t.n_split, a.B, a.hq, a.nq, s);
}

}  // namespace dg
