// MoE router ([P1 二]: 128 experts, 8 per token; [P1 五]: ~84 distinct experts
// touched per 256-token canvas): warp-level top-k of the gate logits with a
// softmax over the selected k, then a deterministic counting sort of the
// (token, slot) items into expert order, the tile work list for the grouped
// expert GEMMs and the count of distinct experts touched.
#include "dg_common.cuh"
#include "kernels.h"

namespace dg {

// One warp per token.  Lane l holds experts l, l+32, ...; k rounds of a warp
// arg-max with (value desc, id asc) ordering pick the top-k.
__global__ void router_topk_kernel(const float* __restrict__ glog, int nsplit, const float* __restrict__ bias,
                                   int32_t* __restrict__ ids, float* __restrict__ wts, int n_tok, int e, int k) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok) return;
  constexpr int kPer = 8;  // E <= 256
  float v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int ex = lane + 32 * j;
    float g = -INFINITY;
    if (ex < e) {
      g = glog[(size_t)warp * e + ex];
      for (int sp = 1; sp < nsplit; ++sp) g += glog[(size_t)sp * n_tok * e + (size_t)warp * e + ex];
      g += bias ? bias[ex] : 0.f;
    }
    v[j] = g;
  }
  float sel_v[16];
  int sel_i[16];
  uint32_t taken = 0;   // bit j: expert lane + 32 j already selected
  for (int r = 0; r < k; ++r) {
    // best local candidate among the experts not yet taken: the first one
    // seen, then strictly larger values (j ascending = id ascending, so the
    // lowest id wins ties, -inf included)
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int ex = lane + 32 * j;
      if (ex < e && !((taken >> j) & 1u) && (bi == 0x7fffffff || v[j] > bv)) { bv = v[j]; bi = ex; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
    }
    // every lane takes lane 0's winner, so the removal below agrees with the output
    bv = __shfl_sync(0xffffffffu, bv, 0);
    bi = __shfl_sync(0xffffffffu, bi, 0);
    sel_v[r] = bv;
    sel_i[r] = bi;
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (lane + 32 * j == bi) taken |= 1u << j;
  }
  if (lane == 0) {
    const float m = sel_v[0];
    float s = 0.f;
    for (int r = 0; r < k; ++r) s += expf(sel_v[r] - m);
    for (int r = 0; r < k; ++r) {
      ids[(size_t)warp * k + r] = sel_i[r];
      wts[(size_t)warp * k + r] = expf(sel_v[r] - m) / s;
    }
  }
}

// Vector form for E = 32 * EPL (EPL a multiple of 4): lane l owns experts
// l*EPL .. l*EPL+EPL-1, read as float4.  The K slices are loaded a group at a
// time (all loads of a group in flight together) and added in slice order,
// so the sums equal the scalar kernel's.
template <int EPL>
__global__ void router_topk_vec_kernel(const float* __restrict__ glog, int nsplit, const float* __restrict__ bias,
                                       int32_t* __restrict__ ids, float* __restrict__ wts, int n_tok, int k) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = 32 * EPL, NV = EPL / 4, G = NV == 1 ? 8 : 4;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok) return;
  const float4* g4 = reinterpret_cast<const float4*>(glog + (size_t)warp * E + lane * EPL);
  const size_t slice4 = (size_t)n_tok * E / 4;
  float v[EPL];
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const float4 a = g4[q];
    v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
  }
  for (int sp0 = 1; sp0 < nsplit; sp0 += G) {
    float4 a[G][NV];
#pragma unroll
    for (int u = 0; u < G; ++u)
#pragma unroll
      for (int q = 0; q < NV; ++q)
        if (sp0 + u < nsplit) a[u][q] = g4[(size_t)(sp0 + u) * slice4 + q];
#pragma unroll
    for (int u = 0; u < G; ++u)
#pragma unroll
      for (int q = 0; q < NV; ++q)
        if (sp0 + u < nsplit) {
          v[4 * q] += a[u][q].x; v[4 * q + 1] += a[u][q].y; v[4 * q + 2] += a[u][q].z; v[4 * q + 3] += a[u][q].w;
        }
  }
  if (bias) {
    const float4* b4 = reinterpret_cast<const float4*>(bias + lane * EPL);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const float4 b = b4[q];
      v[4 * q] += b.x; v[4 * q + 1] += b.y; v[4 * q + 2] += b.z; v[4 * q + 3] += b.w;
    }
  }
  float sel_v[16];
  int sel_i[16];
  uint32_t taken = 0;   // bit j: expert lane * EPL + j already selected
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < EPL; ++j)   // ascending ids: the first of equals wins, -inf included
      if (!((taken >> j) & 1u) && (bi == 0x7fffffff || v[j] > bv)) { bv = v[j]; bi = lane * EPL + j; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
    }
    bv = __shfl_sync(0xffffffffu, bv, 0);
    bi = __shfl_sync(0xffffffffu, bi, 0);
    sel_v[r] = bv;
    sel_i[r] = bi;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane * EPL + j == bi) taken |= 1u << j;
  }
  if (lane == 0) {
    const float m = sel_v[0];
    float s = 0.f;
    for (int r = 0; r < k; ++r) s += expf(sel_v[r] - m);
    for (int r = 0; r < k; ++r) {
      ids[(size_t)warp * k + r] = sel_i[r];
      wts[(size_t)warp * k + r] = expf(sel_v[r] - m) / s;
    }
  }
}

void launch_router_topk(const float* glog, int nsplit, const float* bias, int32_t* ids, float* wts, int n_tok,
                        int e, int k, cudaStream_t s) {
  if (n_tok <= 0) return;
  const int threads = 256;
  const int blocks = (n_tok * 32 + threads - 1) / threads;
  const bool vec = ((uintptr_t)glog & 15u) == 0 && (bias == nullptr || ((uintptr_t)bias & 15u) == 0);
  if (vec && e == 128) {
    launch_k(router_topk_vec_kernel<4>, dim3(blocks), dim3(threads), 0, s, glog, nsplit, bias, ids, wts, n_tok, k);
  } else if (vec && e == 256) {
    launch_k(router_topk_vec_kernel<8>, dim3(blocks), dim3(threads), 0, s, glog, nsplit, bias, ids, wts, n_tok, k);
  } else {
    launch_k(router_topk_kernel, dim3(blocks), dim3(threads), 0, s, glog, nsplit, bias, ids, wts, n_tok, e, k);
  }
}

// Single-CTA counting sort.  Items i = t*k + s in order; inside an expert the
// position of an item is the number of earlier items (smaller i) with the same
// expert, so tokens are ascending and the result needs no atomics in its order.
__global__ void __launch_bounds__(1024) router_permute_kernel(const int32_t* __restrict__ ids, int n_items, int e,
                                                             int tile, int32_t* __restrict__ cnt_out,
                                                             int32_t* __restrict__ off_out,
                                                             int32_t* __restrict__ perm, int32_t* __restrict__ work,
                                                             int32_t* __restrict__ n_work,
                                                             int32_t* __restrict__ touched) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[256];
  __shared__ int off[257];
  __shared__ int running[256];
  __shared__ int wc[32][256];  // per-warp per-expert counts of the current chunk
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int x = tid; x < e; x += blockDim.x) { cnt[x] = 0; running[x] = 0; }
  __syncthreads();
  for (int i = tid; i < n_items; i += blockDim.x) atomicAdd(&cnt[ids[i]], 1);
  __syncthreads();
  if (tid == 0) {
    int acc = 0, nt = 0, nw = 0;
    for (int x = 0; x < e; ++x) {
      off[x] = acc;
      acc += cnt[x];
      if (cnt[x] > 0) ++nt;
      for (int r0 = 0; r0 < cnt[x]; r0 += tile) {
        work[3 * nw + 0] = x;
        work[3 * nw + 1] = off[x] + r0;
        work[3 * nw + 2] = min(tile, cnt[x] - r0);
        ++nw;
      }
    }
    off[e] = acc;
    *n_work = nw;
    *touched = nt;
  }
  __syncthreads();
  for (int x = tid; x < e; x += blockDim.x) cnt_out[x] = cnt[x];
  for (int x = tid; x <= e; x += blockDim.x) off_out[x] = off[x];
  for (int base = 0; base < n_items; base += blockDim.x) {
    for (int x = tid; x < 32 * 256; x += blockDim.x) (&wc[0][0])[x] = 0;
    __syncthreads();
    const int i = base + tid;
    const bool valid = i < n_items;
    const int ex = valid ? ids[i] : -1 - lane;  // invalid lanes never match a real expert
    const unsigned peers = __match_any_sync(0xffffffffu, ex);
    const int lane_rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && lane_rank == 0) wc[w][ex] = __popc(peers);
    __syncthreads();
    // exclusive scan over warps, per expert; advance the running totals
    for (int x = tid; x < e; x += blockDim.x) {
      int acc = running[x];
      for (int ww = 0; ww < 32; ++ww) {
        const int c = wc[ww][x];
        wc[ww][x] = acc;
        acc += c;
      }
      running[x] = acc;
    }
    __syncthreads();
    if (valid) perm[off[ex] + wc[w][ex] + lane_rank] = i;
    __syncthreads();
  }
}

// Single-pass form for up to kPermChunks x 1024 items (a canvas step).  Per
// chunk of 1024 items, each warp counts its items per expert with
// __match_any_sync (no atomics); the per-expert exclusive scan over the 32
// warps (4 threads per expert) gives every item its slot inside its expert,
// kept in registers.  One warp then scans the expert counts into offsets and
// writes the work list with a warp prefix sum, and the items go to
// perm[off[e] + slot].  Same stable order as router_permute_kernel.
constexpr int kPermChunks = 8;

__global__ void __launch_bounds__(1024) router_permute_scan_kernel(const int32_t* __restrict__ ids, int n_items,
                                                                  int e, int tile, int32_t* __restrict__ cnt_out,
                                                                  int32_t* __restrict__ off_out,
                                                                  int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ work,
                                                                  int32_t* __restrict__ n_work,
                                                                  int32_t* __restrict__ touched) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wc[32][256];  // this chunk: per-warp counts, then per-warp exclusive starts
  __shared__ int running[256];
  __shared__ int off[257];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int nch = (n_items + 1023) / 1024;
  for (int x = tid; x < e; x += 1024) running[x] = 0;
  __syncthreads();
  int my_ex[kPermChunks], my_pos[kPermChunks];
#pragma unroll
  for (int c = 0; c < kPermChunks; ++c) {
    my_ex[c] = -1;
    my_pos[c] = 0;
    if (c >= nch) continue;
    const int i = c * 1024 + tid;
    const bool valid = i < n_items;
    const int ex = valid ? ids[i] : -1 - lane;  // invalid lanes never match a real expert
    const unsigned peers = __match_any_sync(0xffffffffu, ex);
    const int rank = __popc(peers & lt);
    for (int x = lane; x < e; x += 32) wc[w][x] = 0;
    __syncwarp();
    if (valid && rank == 0) wc[w][ex] = __popc(peers);
    __syncthreads();
    {
      // exclusive scan over the 32 warps of expert x, 4 threads x 8 warps each
      const int x = tid >> 2, q = tid & 3;
      int sum = 0;
      if (x < e) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = wc[q * 8 + k][x];
          wc[q * 8 + k][x] = sum;
          sum += v;
        }
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o, 4);
        if (q >= o) incl += v;
      }
      if (x < e) {
        const int start = running[x] + incl - sum;
#pragma unroll
        for (int k = 0; k < 8; ++k) wc[q * 8 + k][x] += start;
      }
      __syncthreads();  // every thread has read running[x] before it moves
      if (x < e && q == 3) running[x] += incl;
    }
    __syncthreads();
    if (valid) {
      my_ex[c] = ex;
      my_pos[c] = wc[w][ex] + rank;
    }
  }
  __syncthreads();
  // offsets, tile counts and the work list: warp 0, experts lane*per .. lane*per+per-1
  if (w == 0) {
    const int per = (e + 31) / 32;
    int c_loc = 0, t_loc = 0, nz = 0;
    for (int u = 0; u < per; ++u) {
      const int x = lane * per + u;
      const int c = x < e ? running[x] : 0;
      c_loc += c;
      t_loc += (c + tile - 1) / tile;
      nz += c > 0;
    }
    int c_in = c_loc, t_in = t_loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, c_in, o), b = __shfl_up_sync(0xffffffffu, t_in, o);
      if (lane >= o) { c_in += a; t_in += b; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nz += __shfl_xor_sync(0xffffffffu, nz, o);
    int c_ex = c_in - c_loc, t_ex = t_in - t_loc;
    for (int u = 0; u < per; ++u) {
      const int x = lane * per + u;
      if (x >= e) break;
      const int c = running[x];
      off[x] = c_ex;
      for (int r0 = 0; r0 < c; r0 += tile, ++t_ex) {
        work[3 * t_ex + 0] = x;
        work[3 * t_ex + 1] = c_ex + r0;
        work[3 * t_ex + 2] = min(tile, c - r0);
      }
      c_ex += c;
    }
    if (lane == 31) {
      off[e] = c_in;
      *n_work = t_in;
    }
    if (lane == 0) *touched = nz;
  }
  __syncthreads();
  for (int x = tid; x < e; x += 1024) cnt_out[x] = running[x];
  for (int x = tid; x <= e; x += 1024) off_out[x] = off[x];
#pragma unroll
  for (int c = 0; c < kPermChunks; ++c)
    if (my_ex[c] >= 0) perm[off[my_ex[c]] + my_pos[c]] = c * 1024 + tid;
}

void launch_router_permute(const int32_t* ids, int n_items, int e, int tile, int32_t* cnt, int32_t* off,
                           int32_t* perm, int32_t* work, int32_t* n_work, int32_t* touched, cudaStream_t s) {
  if (n_items <= kPermChunks * 1024 && e <= 256) {
    launch_k(router_permute_scan_kernel, dim3(1), dim3(1024), 0, s, ids, n_items, e, tile, cnt, off, perm, work,
             n_work, touched);
    return;
  }
  launch_k(router_permute_kernel, dim3(1), dim3(1024), 0, s, ids, n_items, e, tile, cnt, off, perm, work, n_work, touched);
}

}  // namespace dg
