// C ABI of the denoising-step library (see include/dg.h) and the host-side
// orchestration of the step: workspaces, KV cache, TMA descriptors, the layer
// loop, the sampler and the block loop with its causal hand-off.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "dg.h"
#include "kernels.h"

using namespace dg;

namespace {

thread_local std::string g_create_error;

// ------------------------------------------------------------ TMA encode
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 map over a row-major [rows, cols] matrix, box (64 cols, box_rows rows), 128-byte swizzle.
bool tmap_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_stride_elems,
             uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// A row-major [rows, cols] bf16 matrix seen as chunks of 64 columns:
// dims (64, rows, cols/64), strides (row pitch, 128 B); box (64, box_rows, nz)
// fetches nz consecutive 64-column chunks of box_rows rows with ONE TMA
// instruction, landing as nz [box_rows x 128 B] 128-byte-swizzled tiles.
// (TMA throughput per CTA grows with the bytes of each instruction.)
bool tmap_chunks(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_pitch_elems,
                 uint32_t box_rows, uint32_t nz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {row_pitch_elems * 2, 128};
  cuuint32_t box[3] = {64, box_rows, nz};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// fp32 output [slices][rows][cols] (row pitch ld elements) for TMA-store
// epilogues: dims (cols, rows, slices), boxes of (128, 32, 1), no swizzle.
// Rows past `rows` of a slice are clipped by the store, never written.
bool tmap_out3d(CUtensorMap* m, void* ptr, uint64_t cols, uint64_t rows, uint64_t slices, uint64_t ld) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, slices};
  cuuint64_t strides[2] = {ld * 4, rows * ld * 4};
  cuuint32_t box[3] = {128, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// Split-attention partial outputs part_o as (256 columns, nq rows, planes):
// boxes of 32 columns x 128 rows x 1 plane, 128-byte swizzle, rows past nq
// clipped by the store.
bool tmap_attn_part(CUtensorMap* m, void* ptr, uint64_t nq, uint64_t planes) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {256, nq, planes};
  cuuint64_t strides[2] = {256 * 4, nq * 256 * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// The same for n2 stacked matrices [n2][rows][cols]: dims (64, rows, cols/64, n2).
bool tmap_chunks4(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t n2, uint32_t box_rows,
                  uint32_t nz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, rows, cols / 64, n2};
  cuuint64_t strides[3] = {cols * 2, 128, cols * rows * 2};
  cuuint32_t box[4] = {64, box_rows, nz, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// uint8 codes of n_mats stacked [rows][K/2] matrices: dims (K/2, rows, n_mats), box (32 bytes, 128 rows, 1),
// no swizzle (the dequantising threads read them row by row).
bool tmap_codes(CUtensorMap* m, const void* ptr, uint64_t half_k, uint64_t rows, uint64_t n_mats) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {half_k, rows, n_mats};
  cuuint64_t strides[2] = {half_k, half_k * rows};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
enum ProfClass {
  PC_EMBED, PC_DENSE, PC_ROPE, PC_ATTN, PC_NORM, PC_ROUTER, PC_GATHER, PC_MOE_UP, PC_MOE_DOWN, PC_COMBINE,
  PC_LMHEAD, PC_SAMPLER, PC_FINISH, PC_COUNT
};
const char* kProfNames[PC_COUNT] = {"embed",  "dense_gemm", "rope_scatter", "attention", "rmsnorm",
                                    "router", "gather",     "moe_up",       "moe_down",  "combine",
                                    "lm_head", "sampler_rows", "sampler_finish"};
static_assert(PC_EMBED == DG_PROF_EMBED && PC_DENSE == DG_PROF_DENSE_GEMM && PC_ROPE == DG_PROF_ROPE_SCATTER &&
                  PC_ATTN == DG_PROF_ATTENTION && PC_NORM == DG_PROF_RMSNORM && PC_ROUTER == DG_PROF_ROUTER &&
                  PC_GATHER == DG_PROF_GATHER && PC_MOE_UP == DG_PROF_MOE_UP && PC_MOE_DOWN == DG_PROF_MOE_DOWN &&
                  PC_COMBINE == DG_PROF_COMBINE && PC_LMHEAD == DG_PROF_LM_HEAD &&
                  PC_SAMPLER == DG_PROF_SAMPLER_ROWS && PC_FINISH == DG_PROF_SAMPLER_FINISH &&
                  PC_COUNT == DG_PROF_COUNT,
              "profiler classes must follow include/dg.h");

}  // namespace

// A weight matrix's TMA maps for 1-, 2- and 4-chunk (64-column) boxes of 128 rows.
struct WMap {
  CUtensorMap k1, k2, k4;
};
struct LayerMaps {
  WMap wq, wk, wv, wo, router, gate, up, down;
  CUtensorMap gate_c, up_c, down_c;   // NVFP4 expert codes
};
struct BMapEntry {
  const void* p;
  uint64_t cols, rows;
  int ntile, ksub;
  CUtensorMap m;
};
struct OMapEntry {
  const void* p;
  uint64_t cols, rows, slices, ld;
  CUtensorMap m;
};

struct dg_handle {
  dg_config c{};
  bool bf16 = false;
  bool fp4 = false;     // expert weights stored as NVFP4
  size_t esz = 4;
  cudaStream_t stream = nullptr;
  int num_sms = 148;
  int dev = 0;
  std::string err;
  // weights (borrowed)
  const void* embed = nullptr;
  const void* w_sc = nullptr;
  const float* final_norm = nullptr;
  std::vector<dg_layer_weights> lw;
  std::vector<LayerMaps> lmaps;
  WMap m_embed{}, m_wsc{};
  std::vector<BMapEntry> bmaps;   // token-operand maps, built on first use
  std::vector<OMapEntry> omaps;   // fp32 output maps of the TMA-store epilogue, built on first use
  struct PartMap {
    int nq, planes;
    CUtensorMap m;
  };
  std::vector<PartMap> part_maps;  // split-attention partial maps by (nq, planes)
  bool bad_launch = false;        // a tensor map or GEMM tiling was rejected
  // KV cache (owned)
  void* kc = nullptr;
  void* vt = nullptr;
  std::vector<int> len;
  // workspace (owned)
  int T_max = 0;
  float* h = nullptr;
  void* xn = nullptr;
  void* eprev = nullptr;
  float* qkv = nullptr;
  void* q = nullptr;
  void* attn = nullptr;
  float* glog = nullptr;
  int32_t* ids = nullptr;
  float* wts = nullptr;
  int32_t* cnt = nullptr;
  int32_t* off = nullptr;
  int32_t* perm = nullptr;
  int32_t* work = nullptr;
  int32_t* n_work = nullptr;
  int n_work_max = 0;
  int32_t* touched = nullptr;
  void* xp = nullptr;
  void* hb = nullptr;
  void* y = nullptr;            // expert outputs [T*k, d] in (token, slot) order, activation type
  float* logits = nullptr;
  VocabStat* vstats = nullptr;  // fused LM head -> sampler: per-token statistics of 32-entry vocabulary groups
  int n_groups = 0;
  float2* rope = nullptr;
  // tensor-core attention (bf16, head dim 256)
  bool attn_tc = false;
  CUtensorMap m_q{};
  std::vector<CUtensorMap> m_kc, m_vt, m_vt2;   // m_vt: boxes of 64 keys x 256 dims; m_vt2: x 128 dims
  float* part_o = nullptr;
  float* part_ml = nullptr;
  size_t part_rows_cap = 0;   // split-rows capacity of part_o / part_ml
  float* kpart = nullptr;      // K-slice partial sums of the split-K dense projections
  size_t kpart_floats = 0;
  // sampler workspace
  void* sws = nullptr;
  int32_t* xh[2] = {nullptr, nullptr};
  int32_t* amax[2] = {nullptr, nullptr};   // argmax rows of two rounds (two-round stop)
  float* mh2[2] = {nullptr, nullptr};      // mean entropies of two rounds (two-round stop)
  float* pmax = nullptr;
  float* ent = nullptr;
  int32_t* keep = nullptr;
  float* meanh = nullptr;
  int32_t* stop = nullptr;
  int32_t* done = nullptr;
  int32_t* canvas = nullptr;
  int32_t* out_tok = nullptr;
  int32_t* req_dev = nullptr;
  int32_t* tok_ws = nullptr;
  int* d_err = nullptr;
  int32_t* h_done = nullptr;  // pinned
  // profiling
  bool prof = false;
  uint32_t prof_mask = 0;
  struct Rec { int cls; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  size_t pool_used = 0;
  uint64_t launches = 0;
};

namespace {

int fail(dg_handle* H, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (H) H->err = buf;
  else g_create_error = buf;
  return code;
}

int cuda_check(dg_handle* H, cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DG_OK;
  return fail(H, DG_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

cudaEvent_t pool_event(dg_handle* H) {
  if (H->pool_used == H->pool.size()) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    H->pool.push_back(e);
  }
  return H->pool[H->pool_used++];
}

struct ProfScope {
  dg_handle* H;
  int cls;
  cudaEvent_t b = nullptr;
  int n;
  bool on;
  ProfScope(dg_handle* h, int c, int n_launch = 1)
      : H(h), cls(c), n(n_launch), on(h->prof && ((h->prof_mask >> c) & 1u)) {
    if (on) {
      cudaEvent_t a = pool_event(H);
      b = pool_event(H);
      cudaEventRecord(a, H->stream);
      H->recs.push_back({cls, a, b});
    }
  }
  ~ProfScope() {
    if (on) cudaEventRecord(b, H->stream);
    H->launches += (uint64_t)n;
  }
};

template <typename T>
T* dalloc(size_t n, bool* ok) {
  void* p = nullptr;
  if (n == 0) n = 1;
  if (cudaMalloc(&p, n * sizeof(T)) != cudaSuccess) { *ok = false; return nullptr; }
  return reinterpret_cast<T*>(p);
}

inline size_t kv_layer_elems(const dg_config& c) {
  return (size_t)c.max_batch * c.n_kv_heads * c.max_ctx * c.head_dim;
}
inline void* kc_layer(dg_handle* H, int l) {
  return (char*)H->kc + (size_t)l * kv_layer_elems(H->c) * H->esz;
}
inline void* vt_layer(dg_handle* H, int l) {
  return (char*)H->vt + (size_t)l * kv_layer_elems(H->c) * H->esz;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int pick_ntile(int n_mtiles, int T, int num_sms) {
  int nt = 256;
  const int tmax = std::max(32, ((T + 31) / 32) * 32);
  while (nt > tmax && nt > 32) nt >>= 1;
  while (nt > 32 && (long)n_mtiles * ((T + nt - 1) / nt) < num_sms) nt >>= 1;
  return nt;
}

// Pipeline shape of the expert GEMMs.  Their K loops are short (down: 11
// chunks), so what counts is latency hidden per SM: single-chunk stages, and
// two co-resident CTAs for the down projection so one CTA's epilogue overlaps
// the other's loads (measured: down 10.0 -> 8.4 ms, gate/up 12.5 -> 12.2 ms
// per full_b1 block against 2-chunk stages and one CTA).
#ifndef DG_MOE_DOWN_KSUB
#define DG_MOE_DOWN_KSUB 1    // 64-column chunks per stage of the expert down projection
#endif
#ifndef DG_MOE_DOWN_CTAS
#define DG_MOE_DOWN_CTAS 2    // co-resident CTAs per SM of the expert down projection
#endif
#ifndef DG_MOE_UP_KSUB
#define DG_MOE_UP_KSUB 1      // chunks per stage of gate/up
#endif
#ifndef DG_MOE_UP_CTAS
#define DG_MOE_UP_CTAS 1      // co-resident CTAs per SM of gate/up
#endif
#ifndef DG_GROUPED_TILE
#define DG_GROUPED_TILE 128   // rows of a tensor-core expert work item (64, 128 or 256)
#endif
// Rows of an expert's work item.  Each item loads a token box sized to its
// rows (32 .. DG_GROUPED_TILE), so a small item does not pay for a large box.
// Larger items stream an expert's weights fewer times but leave fewer items
// to spread over the SMs when the routing concentrates on a few experts.
#ifndef DG_GROUPED_TILE_LARGE
#define DG_GROUPED_TILE_LARGE 256   // rows of an expert work item when a pass has >= DG_LARGE_PASS tokens
#endif
#ifndef DG_LARGE_PASS
#define DG_LARGE_PASS 2048
#endif
int grouped_tile(const dg_handle* H, int T) {
  if (!H->bf16) return 64;
  // the 256-row items are for the CTA-pair kernels; the NVFP4 kernel keeps 128
  if (H->fp4) return DG_GROUPED_TILE;
  return T >= DG_LARGE_PASS ? DG_GROUPED_TILE_LARGE : DG_GROUPED_TILE;
}

// Pipeline shape of a tensor-core GEMM launch.  TMA throughput per CTA is
// set by the bytes of each TMA instruction, so every stage loads each
// operand with one instruction of ksub 64-column chunks: 4 chunks (64 KB of
// weights) for narrow token tiles, 2 chunks when the token tile is wide or
// two weight operands share the stage.
#ifndef DG_NARROW_KSUB
#define DG_NARROW_KSUB 2      // chunks per weight box when the token tile is <= 64 rows
#endif
#ifndef DG_NARROW_CTAS
#define DG_NARROW_CTAS 2      // CTAs per SM when the token tile is <= 64 rows
#endif
#ifndef DG_WIDE_KSUB
#define DG_WIDE_KSUB 1        // chunks per weight box when the token tile is > 64 rows (LM head: 1
                              // chunk, 4 stages measured 16% faster than 2 chunks, 2 stages)
#endif
int ksub_for(int mode, int ntile) { return (mode == 1) ? 2 : (ntile > 64 ? DG_WIDE_KSUB : DG_NARROW_KSUB); }
#ifndef DG_ROUTER_SPLIT
#define DG_ROUTER_SPLIT 16
#endif
constexpr int kMaxKSplit = DG_ROUTER_SPLIT;   // K slices of a split-K projection (router logits)
constexpr int kMaxDenseSplit = 8;      // K slices of the split-K dense projections
constexpr int kDenseSplitRows = 256;   // token rows up to which they take the split-K form
int ctas_for(int ntile) { return ntile <= 64 ? DG_NARROW_CTAS : 1; }

const CUtensorMap& pick(const WMap& w, int ksub) { return ksub == 4 ? w.k4 : ksub == 1 ? w.k1 : w.k2; }

// Token-operand map of a (rows x cols) activation buffer for a tile of ntile
// rows and ksub chunks, built on first use and kept for the handle's life.
const CUtensorMap* bmap(dg_handle* H, const void* p, uint64_t cols, uint64_t rows, int ntile, int ksub) {
  for (const auto& e : H->bmaps)
    if (e.p == p && e.cols == cols && e.rows == rows && e.ntile == ntile && e.ksub == ksub) return &e.m;
  BMapEntry e;
  e.p = p;
  e.cols = cols;
  e.rows = rows;
  e.ntile = ntile;
  e.ksub = ksub;
  if (!tmap_chunks(&e.m, p, cols, rows, cols, (uint32_t)ntile, (uint32_t)ksub)) {
    H->bad_launch = true;
    return nullptr;
  }
  H->bmaps.push_back(e);
  return &H->bmaps.back().m;
}

void run_tc(dg_handle* H, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap* b,
            TcGemm& g, const CUtensorMap* bsub = nullptr, const CUtensorMap* tout = nullptr) {
  if (!b || launch_gemm_tc(a0, a1, a2, *b, bsub, g, H->num_sms, H->stream, tout) != 0) H->bad_launch = true;
}

// Output map of a dense fp32 store (slices of rows x cols, pitch ld), cached;
// returns false when it cannot be built (the launch then uses plain stores).
bool omap(dg_handle* H, void* p, uint64_t cols, uint64_t rows, uint64_t slices, uint64_t ld, CUtensorMap* out) {
  for (const auto& e : H->omaps)
    if (e.p == p && e.cols == cols && e.rows == rows && e.slices == slices && e.ld == ld) {
      *out = e.m;
      return true;
    }
  if (((uintptr_t)p & 15u) != 0 || ld % 4 != 0) return false;
  OMapEntry e;
  e.p = p;
  e.cols = cols;
  e.rows = rows;
  e.slices = slices;
  e.ld = ld;
  if (!tmap_out3d(&e.m, p, cols, rows, slices, ld)) return false;
  if (H->omaps.size() >= 64) H->omaps.clear();   // callers passing fresh output buffers each step
  H->omaps.push_back(e);
  *out = e.m;
  return true;
}

// Token maps of a grouped GEMM's activation rows: boxes of 32, 64 and 128
// rows (bsub) besides the ntile-row map, for work items with fewer rows.
// Returns false when a map could not be built.
bool grouped_bsub(dg_handle* H, const void* x, uint64_t cols, uint64_t rows, int ksub, CUtensorMap bsub[3]) {
  for (int k = 0; k < 3; ++k) {
    const CUtensorMap* m = bmap(H, x, cols, rows, 32 << k, ksub);
    if (!m) return false;
    bsub[k] = *m;
  }
  return true;
}

// ------------------------------------------------------------ GEMM helpers
// out = x[T, K] * W^T (W [n_out, K]) for the dense projections.  With
// max_split > 1 (EPI_STORE_F32 only) K may be split into slices that write
// partial sums at out + s * T * ld_out; returns the number of slices used.
int dense_gemm(dg_handle* H, int cls, const void* x, const void* w, const WMap* mw, int T, int n_out, int K,
               Epi epi, void* out, int ld_out, int max_split = 1) {
  ProfScope ps(H, cls);
  if (!H->bf16) {
    launch_gemm_simt<float>((const float*)x, (const float*)w, T, n_out, K, epi, out, ld_out, nullptr, H->stream);
    return 1;
  }
  TcGemm g{};
  g.mode = 0;
  g.M = n_out;
  g.K = K;
  g.T = T;
  g.ntile = pick_ntile((n_out + 127) / 128, T, H->num_sms);
  g.seg1 = g.seg2 = INT_MAX;
  g.epi = epi;
  g.out = out;
  g.ld_out = ld_out;
  g.err = H->d_err;
  g.ksub = ksub_for(0, g.ntile);
  g.ctas_per_sm = ctas_for(g.ntile);
  // split K (two stages per slice at least) while the grid is below two waves
  const int nst = (K / 64 + g.ksub - 1) / g.ksub;
  const int items = ((n_out + 127) / 128) * ((T + g.ntile - 1) / g.ntile);
  int split = 1;
  if (epi == EPI_STORE_F32 && max_split > 1)
    while (split * 2 <= max_split && split * 2 * 2 <= nst && items * split < 2 * H->num_sms) split *= 2;
  g.ksplit = split;
  g.split_stride = (size_t)T * ld_out;
  const CUtensorMap& a = pick(*mw, g.ksub);
  CUtensorMap to;
  const bool tma_out = epi == EPI_STORE_F32 && omap(H, out, n_out, T, split, ld_out, &to);
  run_tc(H, a, a, a, bmap(H, x, K, H->T_max, g.ntile, g.ksub), g, nullptr, tma_out ? &to : nullptr);
  return split;
}

// Split-K form of a dense projection for up to kDenseSplitRows tokens: the
// token tile holds every row (up to DG_DENSE_MAXN), so each weight tile is
// streamed once, and K is split into slices until the grid fills the SMs.
// Slice s writes its fp32 partial sums to part + s * T * n_out ([T, n_out]
// row-major); the consumer adds the slices in order.  (Adding the slices
// inside a thread-block cluster through distributed shared memory measured
// slower on this part: the partials round-trip through L2 instead.)
#ifndef DG_DENSE_MAXN
#define DG_DENSE_MAXN 256     // token-tile cap (rows of the N operand)
#endif
#ifndef DG_SPLIT_KSUB
#define DG_SPLIT_KSUB 2       // chunks per stage of the split-K dense projections
#endif
struct SplitPlan {
  int ntile = 0, ksub = DG_SPLIT_KSUB, split = 0;
};

SplitPlan split_plan(int num_sms, int T, int n_out, int K, size_t cap_floats) {
  SplitPlan p;
  if (T < 1 || T > kDenseSplitRows || (size_t)T * n_out > cap_floats) return p;
  p.ntile = 32;
  while (p.ntile < T && p.ntile < DG_DENSE_MAXN) p.ntile <<= 1;
  const int nst = (K / 64 + p.ksub - 1) / p.ksub;
  const int tiles = ((n_out + 127) / 128) * ((T + p.ntile - 1) / p.ntile);
  p.split = 1;
  while (p.split < kMaxDenseSplit && tiles * (p.split + 1) <= num_sms && (p.split + 1) * 2 <= nst &&
         (size_t)(p.split + 1) * T * n_out <= cap_floats)
    ++p.split;
  return p;
}

void run_split(dg_handle* H, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2,
               const CUtensorMap* b, int seg1, int seg2, int T, int n_out, int K, const SplitPlan& p, float* part) {
  TcGemm g{};
  g.mode = 0;
  g.M = n_out;
  g.K = K;
  g.T = T;
  g.ntile = p.ntile;
  g.seg1 = seg1;
  g.seg2 = seg2;
  g.epi = EPI_STORE_F32;
  g.out = part;
  g.ld_out = n_out;
  g.err = H->d_err;
  g.ksub = p.ksub;
  g.ctas_per_sm = 1;
  g.ksplit = p.split;
  g.split_stride = (size_t)T * n_out;
  CUtensorMap to;
  const bool tma_out = omap(H, part, n_out, T, p.split, n_out, &to);
  run_tc(H, a0, a1, a2, b, g, nullptr, tma_out ? &to : nullptr);
}

// The split-K form on CTA pairs (k_gemm_tc2.cu): the token tile holds every
// row (64 .. 256), a pair of SMs takes one 256-row weight tile, and K is split
// into as many slices as keep every pair busy in one wave.  Each SM streams
// 128 weight rows and half of the token tile per stage, a third less than a
// single CTA on a 128-row tile, with two 64-column chunks per TMA instruction.
#ifndef DG_DENSE_PAIR
#define DG_DENSE_PAIR 1
#endif
#ifndef DG_PAIR_KSUB
#define DG_PAIR_KSUB 2        // chunks per stage of the CTA-pair dense GEMM
#endif
SplitPlan pair_plan(int num_sms, int T, int n_out, int K, size_t cap_floats, int seg1, int seg2) {
  SplitPlan p;
  if (T < 1 || T > kDenseSplitRows || (size_t)T * n_out > cap_floats) return p;
  if ((seg1 != INT_MAX && seg1 % 256) || (seg2 != INT_MAX && seg2 % 256)) return p;
  p.ksub = DG_PAIR_KSUB;
  p.ntile = 64;
  while (p.ntile < T) p.ntile <<= 1;
  const int nst = (K / 64 + p.ksub - 1) / p.ksub;
  const int items = (n_out + 255) / 256;
  p.split = 1;
  while (p.split < kMaxDenseSplit && items * (p.split + 1) <= num_sms / 2 && (p.split + 1) * 2 <= nst &&
         (size_t)(p.split + 1) * T * n_out <= cap_floats)
    ++p.split;
  return p;
}

// The layers' use of the split-K form: up to three weight maps stacked along
// M (boundaries seg1, seg2), partials in H->kpart.  Returns the number of
// slices, or 0 when the call does not take this form (nothing launched).
int dense_gemm_part(dg_handle* H, int cls, const void* x, const WMap& a0, const WMap& a1, const WMap& a2, int seg1,
                    int seg2, int T, int n_out, int K) {
  if (!H->bf16 || !H->kpart) return 0;
  if (DG_DENSE_PAIR) {
    const SplitPlan q = pair_plan(H->num_sms, T, n_out, K, H->kpart_floats, seg1, seg2);
    if (q.split >= 1) {
      ProfScope ps(H, cls);
      const CUtensorMap* b = bmap(H, x, K, H->T_max, q.ntile / 2, q.ksub);
      TcGemm g{};
      g.mode = 0;
      g.M = n_out;
      g.K = K;
      g.T = T;
      g.ntile = q.ntile;
      g.seg1 = seg1;
      g.seg2 = seg2;
      g.epi = EPI_STORE_F32;
      g.out = H->kpart;
      g.ld_out = n_out;
      g.err = H->d_err;
      g.ksub = q.ksub;
      g.ksplit = q.split;
      g.split_stride = (size_t)T * n_out;
      CUtensorMap to;
      const bool tma_out = omap(H, H->kpart, n_out, T, q.split, n_out, &to);
      if (!b || launch_gemm_tc_pair(pick(a0, q.ksub), pick(a1, q.ksub), pick(a2, q.ksub), *b, g, H->num_sms,
                                    H->stream, tma_out ? &to : nullptr) != 0)
        H->bad_launch = true;
      return q.split;
    }
  }
  const SplitPlan p = split_plan(H->num_sms, T, n_out, K, H->kpart_floats);
  if (p.split < 1) return 0;
  ProfScope ps(H, cls);
  run_split(H, pick(a0, p.ksub), pick(a1, p.ksub), pick(a2, p.ksub), bmap(H, x, K, H->T_max, p.ntile, p.ksub), seg1,
            seg2, T, n_out, K, p, H->kpart);
  return p.split;
}

// q|k|v rows of the layer (fp32 [T, (Hq + 2 Hkv) hd]): returns the number of
// K slices written to H->kpart by the split-K form, or 0 when they are in H->qkv.
int qkv_gemm(dg_handle* H, int l, int T) {
  const dg_config& c = H->c;
  const dg_layer_weights& L = H->lw[l];
  const int nq = c.n_heads * c.head_dim, nk = c.n_kv_heads * c.head_dim;
  const int ld = nq + 2 * nk;
  if (H->bf16) {
    const LayerMaps& M = H->lmaps[l];
    const int ns = dense_gemm_part(H, PC_DENSE, H->xn, M.wq, M.wk, M.wv, nq, nq + nk, T, ld, c.d_model);
    if (ns > 0) return ns;
  }
  ProfScope ps(H, PC_DENSE, H->bf16 ? 1 : 3);
  if (!H->bf16) {
    const float* x = (const float*)H->xn;
    launch_gemm_simt<float>(x, (const float*)L.wq, T, nq, c.d_model, EPI_STORE_F32, H->qkv, ld, nullptr, H->stream);
    launch_gemm_simt<float>(x, (const float*)L.wk, T, nk, c.d_model, EPI_STORE_F32, H->qkv + nq, ld, nullptr,
                            H->stream);
    launch_gemm_simt<float>(x, (const float*)L.wv, T, nk, c.d_model, EPI_STORE_F32, H->qkv + nq + nk, ld, nullptr,
                            H->stream);
    return 0;
  }
  TcGemm g{};
  g.mode = 0;
  g.M = ld;
  g.K = c.d_model;
  g.T = T;
  g.ntile = pick_ntile((ld + 127) / 128, T, H->num_sms);
  g.seg1 = nq;
  g.seg2 = nq + nk;
  g.epi = EPI_STORE_F32;
  g.out = H->qkv;
  g.ld_out = ld;
  g.err = H->d_err;
  g.ksub = ksub_for(0, g.ntile);
  g.ctas_per_sm = ctas_for(g.ntile);
  const LayerMaps& M = H->lmaps[l];
  run_tc(H, pick(M.wq, g.ksub), pick(M.wk, g.ksub), pick(M.wv, g.ksub),
         bmap(H, H->xn, c.d_model, H->T_max, g.ntile, g.ksub), g);
  return 0;
}

void moe_gemms_fp4(dg_handle* H, int l, int T) {
  const dg_config& c = H->c;
  const dg_layer_weights& L = H->lw[l];
  const LayerMaps& M = H->lmaps[l];
  const int tile = grouped_tile(H, T);
  const uint64_t rows = (uint64_t)H->T_max * c.top_k;
  Fp4Gemm g{};
  g.ntile = tile;
  g.work = H->work;
  g.n_work = H->n_work;
  g.n_work_max = c.n_experts + (T * c.top_k + tile - 1) / tile;
  g.err = H->d_err;
  CUtensorMap bsub[3];
  {
    ProfScope ps(H, PC_MOE_UP);
    g.mode = 1;
    g.M = c.d_ff;
    g.K = c.d_model;
    g.out = H->hb;
    g.ld_out = c.d_ff;
    g.sf0 = L.w_gate_sf;
    g.sf1 = L.w_up_sf;
    g.g0 = L.w_gate_g;
    g.g1 = L.w_up_g;
    const CUtensorMap* b = bmap(H, H->xp, c.d_model, rows, tile, 1);
    if (!b || !grouped_bsub(H, H->xp, c.d_model, rows, 1, bsub) ||
        launch_gemm_fp4(M.gate_c, M.up_c, *b, bsub, g, H->num_sms, H->stream) != 0)
      H->bad_launch = true;
  }
  {
    ProfScope ps(H, PC_MOE_DOWN);
    g.mode = 2;
    g.M = c.d_model;
    g.K = c.d_ff;
    g.out = H->y;
    g.ld_out = c.d_model;
    g.row_map = H->perm;
    g.sf0 = L.w_down_sf;
    g.sf1 = nullptr;
    g.g0 = L.w_down_g;
    g.g1 = nullptr;
    const CUtensorMap* b = bmap(H, H->hb, c.d_ff, rows, tile, 1);
    if (!b || !grouped_bsub(H, H->hb, c.d_ff, rows, 1, bsub) ||
        launch_gemm_fp4(M.down_c, M.down_c, *b, bsub, g, H->num_sms, H->stream) != 0)
      H->bad_launch = true;
  }
}

// The grouped GEMMs on CTA pairs (k_moe_tc2.cu): each SM streams 128 weight
// rows and half of an item's token rows.
#ifndef DG_MOE_PAIR
#define DG_MOE_PAIR 1              // bit 0: gate/up on pairs, bit 1: down on pairs (passes below DG_LARGE_PASS)
#endif
#ifndef DG_MOE_PAIR_LARGE
#define DG_MOE_PAIR_LARGE 3        // the same bits for passes of DG_LARGE_PASS tokens or more (256-row items)
#endif
#ifndef DG_MOE_PAIR_MIN_T
#define DG_MOE_PAIR_MIN_T 64       // below this many tokens (AR decode) the one-CTA form keeps more SMs busy per item
#endif
#ifndef DG_MOE_PAIR_UP_KSUB
#define DG_MOE_PAIR_UP_KSUB 1      // chunks per stage, gate/up (two weight operands)
#endif
#ifndef DG_MOE_PAIR_DOWN_KSUB
#define DG_MOE_PAIR_DOWN_KSUB 2    // chunks per stage, down
#endif
// One part (1: gate/up, 2: down) on pairs; false when that part is not run
// this way (nothing launched).
bool moe_gemm_pair(dg_handle* H, int l, int T, int part) {
  const dg_config& c = H->c;
  const int tile = grouped_tile(H, T);
  const bool large = T >= DG_LARGE_PASS;
  if (!H->bf16 || tile > 256 || T < DG_MOE_PAIR_MIN_T || !((large ? DG_MOE_PAIR_LARGE : DG_MOE_PAIR) & part))
    return false;
  const int n_work_max = c.n_experts + (T * c.top_k + tile - 1) / tile;
  const uint64_t rows = (uint64_t)H->T_max * c.top_k;
  const LayerMaps& M = H->lmaps[l];
  TcGemm g{};
  g.ntile = tile;
  g.work = H->work;
  g.n_work = H->n_work;
  g.n_work_max = n_work_max;
  g.err = H->d_err;
  const void* x = part == 1 ? H->xp : H->hb;
  const uint64_t kdim = part == 1 ? c.d_model : c.d_ff;
  g.mode = part;
  g.M = part == 1 ? c.d_ff : c.d_model;
  g.K = (int)kdim;
  g.out = part == 1 ? H->hb : H->y;
  g.ld_out = g.M;
  g.row_map = part == 1 ? nullptr : H->perm;
  g.ksub = part == 1 ? DG_MOE_PAIR_UP_KSUB : DG_MOE_PAIR_DOWN_KSUB;
  const CUtensorMap* b16 = bmap(H, x, kdim, rows, 16, g.ksub);
  const CUtensorMap* b32 = bmap(H, x, kdim, rows, 32, g.ksub);
  const CUtensorMap* b64 = bmap(H, x, kdim, rows, 64, g.ksub);
  const CUtensorMap* b128 = tile > 128 ? bmap(H, x, kdim, rows, 128, g.ksub) : b64;
  const CUtensorMap& a0 = pick(part == 1 ? M.gate : M.down, g.ksub);
  const CUtensorMap& a1 = pick(part == 1 ? M.up : M.down, g.ksub);
  if (!b16 || !b32 || !b64 || !b128 ||
      launch_gemm_tc2_grouped(a0, a1, *b16, *b32, *b64, *b128, g, H->num_sms, H->stream) != 0)
    H->bad_launch = true;
  return true;
}

void moe_gemms(dg_handle* H, int l, int T) {
  if (H->fp4) {
    moe_gemms_fp4(H, l, T);
    return;
  }
  const dg_config& c = H->c;
  const dg_layer_weights& L = H->lw[l];
  const int tile = grouped_tile(H, T);
  const int n_work_max = c.n_experts + (T * c.top_k + tile - 1) / tile;
  const uint64_t rows = (uint64_t)H->T_max * c.top_k;
  {
    ProfScope ps(H, PC_MOE_UP);
    if (moe_gemm_pair(H, l, T, 1)) {
    } else if (!H->bf16) {
      launch_grouped_simt<float>((const float*)H->xp, (const float*)L.w_gate, (const float*)L.w_up, c.d_ff,
                                 c.d_model, H->work, H->n_work, n_work_max, H->perm, true, H->hb, c.d_ff, H->stream);
    } else {
      TcGemm g{};
      g.mode = 1;
      g.M = c.d_ff;
      g.K = c.d_model;
      g.ntile = tile;
      g.seg1 = g.seg2 = INT_MAX;
      g.work = H->work;
      g.n_work = H->n_work;
      g.n_work_max = n_work_max;
      g.epi = EPI_SWIGLU_ACT;
      g.out = H->hb;
      g.ld_out = c.d_ff;
      g.err = H->d_err;
      g.ksub = DG_MOE_UP_KSUB;
      g.ctas_per_sm = DG_MOE_UP_CTAS;
      const LayerMaps& M = H->lmaps[l];
      CUtensorMap bsub[3];
      if (grouped_bsub(H, H->xp, c.d_model, rows, g.ksub, bsub))
        run_tc(H, pick(M.gate, g.ksub), pick(M.up, g.ksub), pick(M.up, g.ksub),
               bmap(H, H->xp, c.d_model, rows, tile, g.ksub), g, bsub);
      else
        H->bad_launch = true;
    }
  }
  {
    ProfScope ps(H, PC_MOE_DOWN);
    if (moe_gemm_pair(H, l, T, 2)) {
    } else if (!H->bf16) {
      launch_grouped_simt<float>((const float*)H->hb, (const float*)L.w_down, nullptr, c.d_model, c.d_ff, H->work,
                                 H->n_work, n_work_max, H->perm, false, H->y, c.d_model, H->stream);
    } else {
      TcGemm g{};
      g.mode = 2;
      g.M = c.d_model;
      g.K = c.d_ff;
      g.ntile = tile;
      g.seg1 = g.seg2 = INT_MAX;
      g.work = H->work;
      g.n_work = H->n_work;
      g.n_work_max = n_work_max;
      g.epi = EPI_SCATTER_ACT;
      g.out = H->y;
      g.ld_out = c.d_model;
      g.row_map = H->perm;
      g.err = H->d_err;
      g.ksub = DG_MOE_DOWN_KSUB;
      g.ctas_per_sm = DG_MOE_DOWN_CTAS;
      const CUtensorMap& a = pick(H->lmaps[l].down, g.ksub);
      CUtensorMap bsub[3];
      if (grouped_bsub(H, H->hb, c.d_ff, rows, g.ksub, bsub))
        run_tc(H, a, a, a, bmap(H, H->hb, c.d_ff, rows, tile, g.ksub), g, bsub);
      else
        H->bad_launch = true;
    }
  }
}

#ifndef DG_ATTN_PAIR
#define DG_ATTN_PAIR 1
#endif
void attention(dg_handle* H, int l, const BatchInfo& bi, int nq, bool causal) {
  const dg_config& c = H->c;
  AttnArgs a{};
  a.B = bi.B;
  a.nq = nq;
  a.hq = c.n_heads;
  a.hkv = c.n_kv_heads;
  a.hd = c.head_dim;
  a.max_ctx = c.max_ctx;
  a.causal = causal ? 1 : 0;
  a.bi = bi;
  if (H->attn_tc && nq == 1) {
    // one new token per request (AR decode): the single-token kernel, GQA heads sharing K/V
    ProfScope ps(H, PC_ATTN, 2);
    if (launch_attn_decode((const __nv_bfloat16*)H->q, (const __nv_bfloat16*)kc_layer(H, l),
                           (const __nv_bfloat16*)vt_layer(H, l), (__nv_bfloat16*)H->attn, a, H->part_o, H->part_ml,
                           H->part_rows_cap, H->num_sms, H->stream) != 0)
      H->bad_launch = true;
    return;
  }
  if (H->attn_tc) {
    // Query heads 2y and 2y+1 on one CTA pair when they read the same KV head
    // (128-key tiles); otherwise one CTA per head (64-key tiles).
    const bool pair = DG_ATTN_PAIR && attn_tc2_supported(c.n_heads, c.n_kv_heads, c.head_dim);
    const int ktile = pair ? 128 : 64;
    // Split the keys: one CTA per SM, so the time is about waves x (key tiles
    // per CTA + a fixed cost of ~2 tiles); each split adds partial-output
    // traffic and combine work (charged half a tile).
    int max_len = 0;
    for (int b = 0; b < bi.B; ++b) max_len = std::max(max_len, bi.len[b] + nq);
    const int base = bi.B * c.n_heads * ((nq + 127) / 128);
    const int tiles = (max_len + ktile - 1) / ktile;
    int n_split = 1;
    double best = 1e30;
    for (int n = 1; n <= std::min(16, std::max(1, tiles / 4)); ++n) {
      const int waves = (base * n + H->num_sms - 1) / H->num_sms;
      const double cost = waves * ((tiles + n - 1) / n + 2.0) + 0.5 * n;
      if (cost < best - 1e-9) { best = cost; n_split = n; }
    }
#ifdef DG_ATTN_SPLIT
    n_split = std::min(DG_ATTN_SPLIT, std::max(1, tiles / 4));   // build-time override for measurements
#endif
    if ((size_t)n_split * bi.B * c.n_heads * nq > H->part_rows_cap) n_split = 1;
    AttnTcArgs t{};
    t.a = a;
    t.n_split = n_split;
    t.part_o = H->part_o;
    t.part_ml = H->part_ml;
    t.nq_pad = nq;
    t.err = H->d_err;
    ProfScope ps(H, PC_ATTN, n_split > 1 ? 2 : 1);
    if (pair) {
      const CUtensorMap* tpo = nullptr;
      if (n_split > 1) {
        const int planes = n_split * bi.B * c.n_heads;
        for (const auto& e : H->part_maps)
          if (e.nq == nq && e.planes == planes) tpo = &e.m;
        if (!tpo) {
          dg_handle::PartMap e;
          e.nq = nq;
          e.planes = planes;
          if (tmap_attn_part(&e.m, H->part_o, (uint64_t)nq, (uint64_t)planes)) {
            if (H->part_maps.size() >= 16) H->part_maps.clear();
            H->part_maps.push_back(e);
            tpo = &H->part_maps.back().m;
          }
        }
      }
      launch_attn_tc2(H->m_q, H->m_kc[l], H->m_vt2[l], tpo, (__nv_bfloat16*)H->attn, t, H->stream);
    }
    else
      launch_attn_tc(H->m_q, H->m_kc[l], H->m_vt[l], (__nv_bfloat16*)H->attn, t, H->stream);
    return;
  }
  ProfScope ps(H, PC_ATTN);
  if (!H->bf16)
    launch_attn_simt<float>((const float*)H->q, (const float*)kc_layer(H, l), (const float*)vt_layer(H, l),
                            (float*)H->attn, a, H->stream);
  else
    launch_attn_simt<__nv_bfloat16>((const __nv_bfloat16*)H->q, (const __nv_bfloat16*)kc_layer(H, l),
                                    (const __nv_bfloat16*)vt_layer(H, l), (__nv_bfloat16*)H->attn, a, H->stream);
}

// The tied LM head with the sampler's first pass in its epilogue: per token and
// 32-entry vocabulary group, (max, first arg-max, sum exp, sum exp * z) of
// z = logit * s / T into H->vstats; the logits themselves are never written.
void lm_head_stats(dg_handle* H, int T, const SamplerArgs& sa) {
  const dg_config& c = H->c;
  ProfScope ps(H, PC_LMHEAD);
  TcGemm g{};
  g.mode = 0;
  g.M = c.vocab;
  g.K = c.d_model;
  g.T = T;
  g.ntile = pick_ntile((c.vocab + 127) / 128, T, H->num_sms);
  g.seg1 = g.seg2 = INT_MAX;
  g.epi = EPI_VOCAB_STATS;
  g.out = H->vstats;
  g.ld_out = 0;
  g.err = H->d_err;
  g.ksub = ksub_for(0, g.ntile);
  g.ctas_per_sm = ctas_for(g.ntile);
  g.argmax_mode = sa.temperature == 0.f ? 1 : 0;
  g.zscale = g.argmax_mode ? sa.logit_scale : sa.logit_scale / sa.temperature;
  g.n_groups = H->n_groups;
  const CUtensorMap& a = pick(H->m_embed, g.ksub);
  run_tc(H, a, a, a, bmap(H, H->xn, c.d_model, H->T_max, g.ntile, g.ksub), g);
}

template <typename T>
void run_layers_t(dg_handle* H, const BatchInfo& bi, int nq, bool causal, const int32_t* tokens,
                  const int32_t* prev, bool head, float* logits, float* hidden_out, const dg_layer_dump* dump,
                  const SamplerArgs* fused) {
  const dg_config& c = H->c;
  const int Tn = bi.B * nq;
  const size_t hbytes = (size_t)Tn * c.d_model * sizeof(float);
  const float eps = (float)c.rms_eps;
  T* xn = (T*)H->xn;
  {
    ProfScope ps(H, PC_EMBED);
    launch_embed<T>(tokens, prev, (const T*)H->embed, H->h, (T*)H->eprev, Tn, c.d_model, c.vocab, H->d_err,
                    H->stream);
  }
  int scs = 0;  // K slices of the self-conditioning term in H->kpart
  if (prev) {
    scs = dense_gemm_part(H, PC_DENSE, H->eprev, H->m_wsc, H->m_wsc, H->m_wsc, INT_MAX, INT_MAX, Tn, c.d_model,
                          c.d_model);
    if (!scs) dense_gemm(H, PC_DENSE, H->eprev, H->w_sc, &H->m_wsc, Tn, c.d_model, c.d_model, EPI_ADD_F32, H->h,
                         c.d_model);
  }
  {
    ProfScope ps(H, PC_NORM);
    const float* w0 = c.n_layers > 0 ? H->lw[0].attn_norm : H->final_norm;
    if (scs) launch_add_rmsnorm<T>(H->h, H->kpart, scs, (size_t)Tn * c.d_model, w0, xn, Tn, c.d_model, eps,
                                   H->stream);
    else launch_rmsnorm<T>(H->h, w0, xn, Tn, c.d_model, eps, H->stream);
  }
  const int ldqkv = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_layer_weights& L = H->lw[l];
    const bool rec = dump && dump->layer == l;
    if (rec && dump->hidden_in) cudaMemcpyAsync(dump->hidden_in, H->h, hbytes, cudaMemcpyDeviceToDevice, H->stream);
    const int qs = qkv_gemm(H, l, Tn);
    {
      ProfScope ps(H, PC_ROPE);
      launch_rope_scatter<T>(qs ? H->kpart : H->qkv, qs ? qs : 1, (size_t)Tn * ldqkv, (T*)H->q, (T*)kc_layer(H, l),
                             (T*)vt_layer(H, l), (const float*)H->rope, bi, nq, c.n_heads, c.n_kv_heads, c.head_dim,
                             c.max_ctx, H->stream);
    }
    attention(H, l, bi, nq, causal);
    const int nqc = c.n_heads * c.head_dim;
    const int os = H->bf16 ? dense_gemm_part(H, PC_DENSE, H->attn, H->lmaps[l].wo, H->lmaps[l].wo, H->lmaps[l].wo,
                                             INT_MAX, INT_MAX, Tn, c.d_model, nqc)
                           : 0;
    if (!os) dense_gemm(H, PC_DENSE, H->attn, L.wo, H->bf16 ? &H->lmaps[l].wo : nullptr, Tn, c.d_model, nqc,
                        EPI_ADD_F32, H->h, c.d_model);
    {
      ProfScope ps(H, PC_NORM);
      if (os) launch_add_rmsnorm<T>(H->h, H->kpart, os, (size_t)Tn * c.d_model, L.ffn_norm, xn, Tn, c.d_model, eps,
                                    H->stream);
      else launch_rmsnorm<T>(H->h, L.ffn_norm, xn, Tn, c.d_model, eps, H->stream);
    }
    // the router projection has one 128-row weight tile: split K for parallelism
    const int rsplit = dense_gemm(H, PC_ROUTER, H->xn, L.router_w, H->bf16 ? &H->lmaps[l].router : nullptr, Tn,
                                  c.n_experts, c.d_model, EPI_STORE_F32, H->glog, c.n_experts, kMaxKSplit);
    {
      ProfScope ps(H, PC_ROUTER, 2);
      launch_router_topk(H->glog, rsplit, L.router_b, H->ids, H->wts, Tn, c.n_experts, c.top_k, H->stream);
      launch_router_permute(H->ids, Tn * c.top_k, c.n_experts, grouped_tile(H, Tn), H->cnt, H->off, H->perm,
                            H->work, H->n_work, H->touched + l, H->stream);
    }
    if (rec && dump->expert_ids)
      cudaMemcpyAsync(dump->expert_ids, H->ids, (size_t)Tn * c.top_k * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      H->stream);
    if (rec && dump->expert_wts)
      cudaMemcpyAsync(dump->expert_wts, H->wts, (size_t)Tn * c.top_k * sizeof(float), cudaMemcpyDeviceToDevice,
                      H->stream);
    {
      ProfScope ps(H, PC_GATHER);
      launch_gather_rows<T>(xn, H->perm, (T*)H->xp, Tn * c.top_k, c.top_k, c.d_model, H->stream);
    }
    moe_gemms(H, l, Tn);
    {
      ProfScope ps(H, PC_COMBINE);
      const float* nw = (l + 1 < c.n_layers) ? H->lw[l + 1].attn_norm : (head ? H->final_norm : nullptr);
      if (hidden_out && l + 1 == c.n_layers) nw = nullptr;
      launch_combine<T>(H->h, (const T*)H->y, H->wts, c.top_k, nw, xn, Tn, c.d_model, eps, H->stream);
    }
    if (rec && dump->hidden_out) cudaMemcpyAsync(dump->hidden_out, H->h, hbytes, cudaMemcpyDeviceToDevice, H->stream);
  }
  if (hidden_out) {
    cudaMemcpyAsync(hidden_out, H->h, hbytes, cudaMemcpyDeviceToDevice, H->stream);
    if (head) {
      ProfScope ps(H, PC_NORM);
      launch_rmsnorm<T>(H->h, H->final_norm, xn, Tn, c.d_model, eps, H->stream);
    }
  }
  if (head && fused) lm_head_stats(H, Tn, *fused);
  else if (head) dense_gemm(H, PC_LMHEAD, H->xn, H->embed, &H->m_embed, Tn, c.vocab, c.d_model, EPI_STORE_F32,
                            logits, c.vocab);
}

void run_layers(dg_handle* H, const BatchInfo& bi, int nq, bool causal, const int32_t* tokens, const int32_t* prev,
                bool head, float* logits, float* hidden_out, const dg_layer_dump* dump = nullptr,
                const SamplerArgs* fused = nullptr) {
  if (H->bf16) run_layers_t<__nv_bfloat16>(H, bi, nq, causal, tokens, prev, head, logits, hidden_out, dump, fused);
  else run_layers_t<float>(H, bi, nq, causal, tokens, prev, head, logits, hidden_out, dump, nullptr);
}

int make_batch(dg_handle* H, int batch, const int* req, BatchInfo* bi) {
  if (batch < 1 || batch > H->c.max_batch || !req) return fail(H, DG_EINVAL, "batch %d out of range [1,%d]", batch,
                                                               H->c.max_batch);
  bi->B = batch;
  for (int b = 0; b < batch; ++b) {
    if (req[b] < 0 || req[b] >= H->c.max_batch) return fail(H, DG_EINVAL, "request slot %d out of range", req[b]);
    for (int x = 0; x < b; ++x)
      if (req[x] == req[b]) return fail(H, DG_EINVAL, "request slot %d repeated in a batch", req[b]);
    bi->slot[b] = req[b];
    bi->len[b] = H->len[req[b]];
  }
  return DG_OK;
}

int upload_req(dg_handle* H, const BatchInfo& bi) {
  int32_t tmp[kMaxBatch];
  for (int b = 0; b < bi.B; ++b) tmp[b] = bi.slot[b];
  // pageable copy: the staging buffer is on the stack, so the runtime copies synchronously
  return cuda_check(H, cudaMemcpyAsync(H->req_dev, tmp, bi.B * sizeof(int32_t), cudaMemcpyHostToDevice, H->stream),
                    "upload request ids");
}

int check_launch(dg_handle* H, const char* what) {
  if (H->bad_launch) {
    H->bad_launch = false;
    return fail(H, DG_ECUDA, "%s: a tensor map or GEMM tiling was rejected (nothing was launched for it)", what);
  }
  return cuda_check(H, cudaGetLastError(), what);
}

SamplerArgs sampler_args(const dg_sampler_params& sp, int step) {
  SamplerArgs a;
  a.temperature = sp.temperature;
  a.logit_scale = sp.logit_scale;
  a.stop_threshold = sp.stop_threshold;
  a.keep_k = sp.keep_k;
  a.seed = sp.seed;
  a.block = sp.block;
  a.step = (uint32_t)step;
  a.keep_mode = sp.keep_mode;
  a.entropy_budget = sp.entropy_budget;
  a.stop_mode = sp.stop_mode;
  a.prev_argmax = sp.prev_argmax;
  a.prev_mean_h = sp.prev_mean_entropy;
  return a;
}

int check_sampler_params(dg_handle* H, const dg_sampler_params* sp) {
  if (!sp) return fail(H, DG_EINVAL, "null sampler params");
  if (!(sp->temperature >= 0.f) || !std::isfinite(sp->temperature))
    return fail(H, DG_EINVAL, "temperature must be finite and >= 0");
  if (!(sp->logit_scale > 0.f) || !std::isfinite(sp->logit_scale)) return fail(H, DG_EINVAL, "logit_scale must be > 0");
  if (sp->keep_k < 0 || sp->keep_k > H->c.canvas) return fail(H, DG_EINVAL, "keep_k out of [0, N]");
  if (sp->keep_mode != DG_KEEP_TOPK && sp->keep_mode != DG_KEEP_ENTROPY_BUDGET)
    return fail(H, DG_EINVAL, "unknown keep_mode %d", sp->keep_mode);
  if (sp->keep_mode == DG_KEEP_ENTROPY_BUDGET && !(sp->entropy_budget >= 0.f && std::isfinite(sp->entropy_budget)))
    return fail(H, DG_EINVAL, "entropy_budget must be finite and >= 0");
  if (sp->stop_mode != DG_STOP_MEAN_ENTROPY && sp->stop_mode != DG_STOP_TWO_ROUNDS)
    return fail(H, DG_EINVAL, "unknown stop_mode %d", sp->stop_mode);
  return DG_OK;
}

// sampler over logits rows of the batch, then keep / re-noise / stop
// logits == nullptr: the fused form, from the LM head's group statistics in H->vstats
void run_sampler(dg_handle* H, const float* logits, const BatchInfo& bi, const SamplerArgs& a, int32_t* canvas,
                 int32_t* xh, float* pmax, float* ent, int32_t* keep, float* meanh, int32_t* stop, int32_t* done,
                 int32_t* out_tokens, int final_step, int32_t* argmax) {
  const int n = H->c.canvas;
  if (!logits) {
    ProfScope ps(H, PC_SAMPLER, 1);
    launch_sampler_fused_rows(H->vstats, H->n_groups, (const __nv_bfloat16*)H->xn, (const __nv_bfloat16*)H->embed,
                              H->c.d_model, bi.B * n, n, H->c.vocab, H->req_dev, a, xh, pmax, ent, H->stream, argmax);
  } else {
    ProfScope ps(H, PC_SAMPLER, 2);
    launch_sampler_rows(logits, bi.B * n, n, H->c.vocab, H->req_dev, a, H->sws, xh, pmax, ent, H->stream, argmax);
  }
  {
    ProfScope ps(H, PC_FINISH);
    launch_sampler_finish(xh, pmax, ent, bi.B, n, H->c.vocab, H->req_dev, a, canvas, keep, meanh, stop, done,
                          out_tokens, final_step, H->stream, argmax);
  }
}

int read_device_error(dg_handle* H) {
  int e = 0;
  if (cudaMemcpy(&e, H->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(H, DG_ECUDA, "reading the device error flag: %s", cudaGetErrorString(cudaGetLastError()));
  if (e != 0) {
    cudaMemset(H->d_err, 0, sizeof(int));
    if (e == 5) return fail(H, DG_EINVAL, "a token outside [0, vocab) reached the embedding (replaced by 0)");
    return fail(H, DG_ETIMEOUT, "a bounded device wait gave up (code %d)", e);
  }
  return DG_OK;
}

int encode_causal(dg_handle* H, const BatchInfo& bi0, const int32_t* tokens, int n, int src_pitch) {
  // chunked causal encode: B * chunk <= T_max
  BatchInfo bi = bi0;
  const int chunk = std::max(1, std::min(n, H->T_max / bi.B));
  for (int p0 = 0; p0 < n; p0 += chunk) {
    const int m = std::min(chunk, n - p0);
    if (cudaMemcpy2DAsync(H->tok_ws, m * sizeof(int32_t), tokens + p0, src_pitch * sizeof(int32_t),
                          m * sizeof(int32_t), bi.B, cudaMemcpyDeviceToDevice, H->stream) != cudaSuccess)
      return fail(H, DG_ECUDA, "token staging copy failed");
    run_layers(H, bi, m, true, H->tok_ws, nullptr, false, nullptr, nullptr);
    int rc = check_launch(H, "causal encode");
    if (rc) return rc;
    for (int b = 0; b < bi.B; ++b) {
      bi.len[b] += m;
      H->len[bi.slot[b]] += m;
    }
  }
  return DG_OK;
}

}  // namespace

// ======================================================================= ABI

extern "C" {

const char* dg_last_error(const dg_handle* h) { return h ? h->err.c_str() : g_create_error.c_str(); }

int dg_create(const dg_config* cfg, const dg_weights* w, void* stream, dg_handle** out) {
  g_create_error.clear();
  if (!cfg || !out) return fail(nullptr, DG_EINVAL, "null config or output pointer");
  *out = nullptr;
  const dg_config& c = *cfg;
  if (c.dtype != DG_FP32 && c.dtype != DG_BF16) return fail(nullptr, DG_EINVAL, "dtype must be DG_FP32 or DG_BF16");
  if (c.n_layers < 0 || c.canvas < 1 || c.canvas > 1024 || c.vocab < 1 || c.max_batch < 1 ||
      c.max_batch > kMaxBatch)
    return fail(nullptr, DG_EINVAL, "bad layers/canvas/vocab/max_batch");
  const bool model = c.n_layers > 0;
  if (model) {
    if (c.d_model < 1 || c.n_heads < 1 || c.n_kv_heads < 1 || c.n_heads % c.n_kv_heads || c.head_dim < 2 ||
        c.head_dim % 2 || c.head_dim > 256 || c.n_experts < 1 || c.n_experts > 256 || c.top_k < 1 ||
        c.top_k > 16 || c.top_k > c.n_experts || c.d_ff < 1)
      return fail(nullptr, DG_EINVAL, "bad model shape");
    if (8 % (c.n_heads / c.n_kv_heads) != 0) return fail(nullptr, DG_EINVAL, "Hq/Hkv must divide 8");
    if (c.max_ctx < c.canvas || c.max_ctx % 64) return fail(nullptr, DG_EINVAL, "max_ctx must be a multiple of 64 >= canvas");
    if (!(c.rms_eps > 0) || !(c.rope_base > 1)) return fail(nullptr, DG_EINVAL, "bad rms_eps / rope_base");
    if (c.dtype == DG_BF16 && (c.d_model % 64 || c.d_ff % 64 || c.head_dim % 64))
      return fail(nullptr, DG_EINVAL, "bf16 needs d_model, d_ff, head_dim multiples of 64");
    if (c.expert_format != DG_EXPERT_DTYPE && c.expert_format != DG_EXPERT_NVFP4)
      return fail(nullptr, DG_EINVAL, "unknown expert_format %d", c.expert_format);
    if (c.expert_format == DG_EXPERT_NVFP4 && c.dtype != DG_BF16)
      return fail(nullptr, DG_EINVAL, "NVFP4 experts need a bf16 handle");
    if (!w || !w->embed || !w->w_sc || !w->final_norm || !w->layers)
      return fail(nullptr, DG_EINVAL, "null weight pointer");
    if (!aligned16(w->final_norm)) return fail(nullptr, DG_EINVAL, "unaligned final_norm");
    for (int l = 0; l < c.n_layers; ++l) {
      const dg_layer_weights& L = w->layers[l];
      const void* ps[] = {L.attn_norm, L.wq, L.wk, L.wv, L.wo, L.ffn_norm, L.router_w, L.w_gate, L.w_up, L.w_down};
      for (const void* p : ps)
        if (!p || !aligned16(p)) return fail(nullptr, DG_EINVAL, "layer %d: null or unaligned weight", l);
      if (c.expert_format == DG_EXPERT_NVFP4) {
        const void* qs[] = {L.w_gate_sf, L.w_up_sf, L.w_down_sf, L.w_gate_g, L.w_up_g, L.w_down_g};
        for (const void* p : qs)
          if (!p || !aligned16(p)) return fail(nullptr, DG_EINVAL, "layer %d: null or unaligned NVFP4 scales", l);
      }
    }
    if (!aligned16(w->embed) || !aligned16(w->w_sc)) return fail(nullptr, DG_EINVAL, "unaligned embed / w_sc");
    // the router needs finite gate logits: a non-finite bias is refused here
    std::vector<float> bias_h(c.n_experts);
    for (int l = 0; l < c.n_layers; ++l) {
      if (!w->layers[l].router_b) continue;
      if (cudaMemcpy(bias_h.data(), w->layers[l].router_b, c.n_experts * sizeof(float), cudaMemcpyDeviceToHost) !=
          cudaSuccess)
        return fail(nullptr, DG_EINVAL, "layer %d: router_b is not a readable device pointer (%s)", l,
                    cudaGetErrorString(cudaGetLastError()));
      for (float b : bias_h)
        if (!std::isfinite(b)) return fail(nullptr, DG_EINVAL, "layer %d: router_b holds a non-finite value", l);
    }
  }
  dg_handle* H = new dg_handle();
  H->c = c;
  if (H->c.max_tokens <= 0) H->c.max_tokens = c.max_batch * c.canvas;
  if (H->c.max_tokens < c.max_batch * c.canvas) {
    delete H;
    return fail(nullptr, DG_EINVAL, "max_tokens < max_batch * canvas");
  }
  H->bf16 = c.dtype == DG_BF16;
  H->fp4 = model && c.expert_format == DG_EXPERT_NVFP4;
  H->esz = H->bf16 ? 2 : 4;
  H->stream = (cudaStream_t)stream;
  cudaGetDevice(&H->dev);
  cudaDeviceGetAttribute(&H->num_sms, cudaDevAttrMultiProcessorCount, H->dev);
  H->len.assign(c.max_batch, 0);
  H->T_max = H->c.max_tokens;
  bool ok = true;
  const int T = H->T_max;
  const int nrow = c.max_batch * c.canvas;
  if (model) {
    H->embed = w->embed;
    H->w_sc = w->w_sc;
    H->final_norm = w->final_norm;
    H->lw.assign(w->layers, w->layers + c.n_layers);
    const size_t kvn = kv_layer_elems(c) * c.n_layers;
    H->kc = dalloc<char>(kvn * H->esz, &ok);
    H->vt = dalloc<char>(kvn * H->esz, &ok);
    const int qw = c.n_heads * c.head_dim;
    const int ldqkv = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
    H->h = dalloc<float>((size_t)T * c.d_model, &ok);
    H->xn = dalloc<char>((size_t)T * c.d_model * H->esz, &ok);
    H->eprev = dalloc<char>((size_t)T * c.d_model * H->esz, &ok);
    H->qkv = dalloc<float>((size_t)T * ldqkv, &ok);
    H->q = dalloc<char>((size_t)T * qw * H->esz, &ok);
    H->attn = dalloc<char>((size_t)T * qw * H->esz, &ok);
    H->glog = dalloc<float>((size_t)T * c.n_experts * kMaxKSplit, &ok);
    H->ids = dalloc<int32_t>((size_t)T * c.top_k, &ok);
    H->wts = dalloc<float>((size_t)T * c.top_k, &ok);
    H->cnt = dalloc<int32_t>(c.n_experts, &ok);
    H->off = dalloc<int32_t>(c.n_experts + 1, &ok);
    H->perm = dalloc<int32_t>((size_t)T * c.top_k, &ok);
    H->n_work_max = c.n_experts + (T * c.top_k + 63) / 64;
    H->work = dalloc<int32_t>((size_t)3 * H->n_work_max, &ok);
    H->n_work = dalloc<int32_t>(1, &ok);
    H->touched = dalloc<int32_t>(c.n_layers, &ok);
    H->xp = dalloc<char>((size_t)T * c.top_k * c.d_model * H->esz, &ok);
    H->hb = dalloc<char>((size_t)T * c.top_k * c.d_ff * H->esz, &ok);
    H->y = dalloc<char>((size_t)T * c.top_k * c.d_model * H->esz, &ok);
    H->logits = dalloc<float>((size_t)nrow * c.vocab, &ok);
    if (c.dtype == DG_BF16) {
      H->n_groups = (c.vocab + 31) / 32;
      H->vstats = dalloc<VocabStat>((size_t)nrow * H->n_groups, &ok);
    }
    H->rope = dalloc<float2>((size_t)c.max_ctx * (c.head_dim / 2), &ok);
    H->tok_ws = dalloc<int32_t>((size_t)T, &ok);
    if (c.dtype == DG_BF16) {
      H->kpart_floats = (size_t)kMaxDenseSplit * std::min(T, kDenseSplitRows) * std::max(ldqkv, c.d_model);
      H->kpart = dalloc<float>(H->kpart_floats, &ok);
    }
    if (c.dtype == DG_BF16 && c.head_dim == 256) {
      H->part_rows_cap = (size_t)16 * c.canvas * c.n_heads;
      H->part_o = dalloc<float>(H->part_rows_cap * c.head_dim, &ok);
      H->part_ml = dalloc<float>(H->part_rows_cap * 2, &ok);
    }
  }
  H->sws = dalloc<char>(sampler_workspace_bytes(nrow, c.vocab), &ok);
  H->xh[0] = dalloc<int32_t>(nrow, &ok);
  H->xh[1] = dalloc<int32_t>(nrow, &ok);
  H->amax[0] = dalloc<int32_t>(nrow, &ok);
  H->amax[1] = dalloc<int32_t>(nrow, &ok);
  H->mh2[0] = dalloc<float>(c.max_batch, &ok);
  H->mh2[1] = dalloc<float>(c.max_batch, &ok);
  H->pmax = dalloc<float>(nrow, &ok);
  H->ent = dalloc<float>(nrow, &ok);
  H->keep = dalloc<int32_t>(nrow, &ok);
  H->meanh = dalloc<float>(c.max_batch, &ok);
  H->stop = dalloc<int32_t>(c.max_batch, &ok);
  H->done = dalloc<int32_t>(c.max_batch, &ok);
  H->canvas = dalloc<int32_t>(nrow, &ok);
  H->out_tok = dalloc<int32_t>(nrow, &ok);
  H->req_dev = dalloc<int32_t>(c.max_batch, &ok);
  H->d_err = dalloc<int>(1, &ok);
  if (cudaMallocHost(&H->h_done, c.max_batch * sizeof(int32_t)) != cudaSuccess) ok = false;
  if (!ok) {
    dg_destroy(H);
    cudaGetLastError();
    return fail(nullptr, DG_ENOMEM, "device allocation failed");
  }
  cudaMemset(H->d_err, 0, sizeof(int));
  if (model) {
    const size_t kvn = kv_layer_elems(c) * c.n_layers;
    cudaMemset(H->kc, 0, kvn * H->esz);
    cudaMemset(H->vt, 0, kvn * H->esz);
    // RoPE table: (cos, sin) of pos * base^(-2j/hd), in double on the host
    const int half = c.head_dim / 2;
    std::vector<float2> tab((size_t)c.max_ctx * half);
    for (int p = 0; p < c.max_ctx; ++p)
      for (int j = 0; j < half; ++j) {
        const double th = std::pow(c.rope_base, -2.0 * j / c.head_dim);
        const double ang = (double)p * th;
        tab[(size_t)p * half + j] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    cudaMemcpy(H->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (H->bf16) {
      const int d = c.d_model, F = c.d_ff, E = c.n_experts;
      const int qw = c.n_heads * c.head_dim, kw = c.n_kv_heads * c.head_dim;
      bool tm = true;
      H->lmaps.resize(c.n_layers);
      for (int l = 0; l < c.n_layers; ++l) {
        const dg_layer_weights& L = H->lw[l];
        LayerMaps& M = H->lmaps[l];
        auto dense = [&](WMap& w, const void* p, uint64_t cols, uint64_t rows) {
          tm &= tmap_chunks(&w.k1, p, cols, rows, cols, 128, 1);
          tm &= tmap_chunks(&w.k2, p, cols, rows, cols, 128, 2);
          tm &= tmap_chunks(&w.k4, p, cols, rows, cols, 128, 4);
        };
        auto experts = [&](WMap& w, const void* p, uint64_t cols, uint64_t rows) {
          tm &= tmap_chunks4(&w.k1, p, cols, rows, E, 128, 1);
          tm &= tmap_chunks4(&w.k2, p, cols, rows, E, 128, 2);
          tm &= tmap_chunks4(&w.k4, p, cols, rows, E, 128, 4);
        };
        dense(M.wq, L.wq, d, qw);
        dense(M.wk, L.wk, d, kw);
        dense(M.wv, L.wv, d, kw);
        dense(M.wo, L.wo, qw, d);
        dense(M.router, L.router_w, d, E);
        if (H->fp4) {
          tm &= tmap_codes(&M.gate_c, L.w_gate, d / 2, F, E);
          tm &= tmap_codes(&M.up_c, L.w_up, d / 2, F, E);
          tm &= tmap_codes(&M.down_c, L.w_down, F / 2, d, E);
        } else {
          experts(M.gate, L.w_gate, d, F);
          experts(M.up, L.w_up, d, F);
          experts(M.down, L.w_down, F, d);
        }
      }
      tm &= tmap_chunks(&H->m_embed.k1, H->embed, d, c.vocab, d, 128, 1);
      tm &= tmap_chunks(&H->m_embed.k2, H->embed, d, c.vocab, d, 128, 2);
      tm &= tmap_chunks(&H->m_embed.k4, H->embed, d, c.vocab, d, 128, 4);
      tm &= tmap_chunks(&H->m_wsc.k1, H->w_sc, d, d, d, 128, 1);
      tm &= tmap_chunks(&H->m_wsc.k2, H->w_sc, d, d, d, 128, 2);
      tm &= tmap_chunks(&H->m_wsc.k4, H->w_sc, d, d, d, 128, 4);
      if (c.head_dim == 256) {
        H->attn_tc = true;
        const uint64_t hd = (uint64_t)c.head_dim;
        tm &= tmap_chunks(&H->m_q, H->q, hd, (uint64_t)T * c.n_heads, hd, 128, 4);
        H->m_kc.resize(c.n_layers);
        H->m_vt.resize(c.n_layers);
        H->m_vt2.resize(c.n_layers);
        const uint64_t kv_rows = (uint64_t)c.max_batch * c.n_kv_heads;
        for (int l = 0; l < c.n_layers; ++l) {
          tm &= tmap_chunks(&H->m_kc[l], kc_layer(H, l), hd, kv_rows * c.max_ctx, hd, 64, 4);
          tm &= tmap_2d(&H->m_vt[l], vt_layer(H, l), (uint64_t)c.max_ctx, kv_rows * hd, (uint64_t)c.max_ctx, 256);
          tm &= tmap_2d(&H->m_vt2[l], vt_layer(H, l), (uint64_t)c.max_ctx, kv_rows * hd, (uint64_t)c.max_ctx, 128);
        }
      }
      if (!tm) {
        dg_destroy(H);
        return fail(nullptr, DG_ECUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
      }
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    const char* m = cudaGetErrorString(cudaGetLastError());
    dg_destroy(H);
    return fail(nullptr, DG_ECUDA, "create: %s", m);
  }
  *out = H;
  return DG_OK;
}

void dg_destroy(dg_handle* H) {
  if (!H) return;
  cudaStreamSynchronize(H->stream);  // the legacy default stream when the handle has none
  void* ps[] = {H->kc, H->vt, H->h, H->xn, H->eprev, H->qkv, H->q, H->attn, H->glog, H->ids, H->wts, H->cnt,
                H->off, H->perm, H->work, H->n_work, H->touched, H->xp, H->hb, H->y, H->logits, H->rope, H->sws,
                H->xh[0], H->xh[1], H->pmax, H->ent, H->keep, H->meanh, H->stop, H->done, H->canvas, H->out_tok,
                H->req_dev, H->tok_ws, H->d_err, H->part_o, H->part_ml, H->kpart, H->amax[0], H->amax[1],
                H->mh2[0], H->mh2[1], H->vstats};
  for (void* p : ps)
    if (p) cudaFree(p);
  if (H->h_done) cudaFreeHost(H->h_done);
  for (cudaEvent_t e : H->pool) cudaEventDestroy(e);
  delete H;
}

int dg_set_length(dg_handle* H, int req, int length) {
  if (!H) return DG_EINVAL;
  if (req < 0 || req >= H->c.max_batch) return fail(H, DG_EINVAL, "request slot out of range");
  if (length < 0 || length > H->c.max_ctx) return fail(H, DG_ECAPACITY, "length %d exceeds max_ctx", length);
  H->len[req] = length;
  return DG_OK;
}

int dg_get_length(const dg_handle* H, int req, int* length) {
  if (!H || !length || req < 0 || req >= H->c.max_batch) return DG_EINVAL;
  *length = H->len[req];
  return DG_OK;
}

int dg_set_kv(dg_handle* H, int req, int layer, const void* k, const void* v, int n) {
  if (!H) return DG_EINVAL;
  const dg_config& c = H->c;
  if (c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  if (req < 0 || req >= c.max_batch || layer < 0 || layer >= c.n_layers || !k || !v || n < 0)
    return fail(H, DG_EINVAL, "bad set_kv arguments");
  if (n > c.max_ctx) return fail(H, DG_ECAPACITY, "n exceeds max_ctx");
  const size_t slot_off = (size_t)req * c.n_kv_heads * c.max_ctx * c.head_dim * H->esz;
  char* kc = (char*)kc_layer(H, layer) + slot_off;
  char* vt = (char*)vt_layer(H, layer) + slot_off;
  if (H->bf16)
    launch_set_kv<__nv_bfloat16>((const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (__nv_bfloat16*)kc,
                                 (__nv_bfloat16*)vt, c.n_kv_heads, n, c.head_dim, c.max_ctx, H->stream);
  else
    launch_set_kv<float>((const float*)k, (const float*)v, (float*)kc, (float*)vt, c.n_kv_heads, n, c.head_dim,
                         c.max_ctx, H->stream);
  H->launches += 1;
  return check_launch(H, "set_kv");
}

int dg_get_kv(dg_handle* H, int req, int layer, void* k, void* v, int n) {
  if (!H) return DG_EINVAL;
  const dg_config& c = H->c;
  if (c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  if (req < 0 || req >= c.max_batch || layer < 0 || layer >= c.n_layers || !k || !v || n < 0)
    return fail(H, DG_EINVAL, "bad get_kv arguments");
  if (n > c.max_ctx) return fail(H, DG_ECAPACITY, "n exceeds max_ctx");
  const size_t slot_off = (size_t)req * c.n_kv_heads * c.max_ctx * c.head_dim * H->esz;
  const char* kc = (const char*)kc_layer(H, layer) + slot_off;
  const char* vt = (const char*)vt_layer(H, layer) + slot_off;
  if (H->bf16)
    launch_get_kv<__nv_bfloat16>((const __nv_bfloat16*)kc, (const __nv_bfloat16*)vt, (__nv_bfloat16*)k,
                                 (__nv_bfloat16*)v, c.n_kv_heads, n, c.head_dim, c.max_ctx, H->stream);
  else
    launch_get_kv<float>((const float*)kc, (const float*)vt, (float*)k, (float*)v, c.n_kv_heads, n, c.head_dim,
                         c.max_ctx, H->stream);
  H->launches += n > 0 ? 1 : 0;
  return check_launch(H, "get_kv");
}

int dg_prefill_prompt(dg_handle* H, int batch, const int* req, const int32_t* tokens, int n) {
  if (!H) return DG_EINVAL;
  if (H->c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  if (!tokens || n < 0) return fail(H, DG_EINVAL, "bad tokens");
  BatchInfo bi;
  int rc = make_batch(H, batch, req, &bi);
  if (rc) return rc;
  for (int b = 0; b < batch; ++b)
    if (bi.len[b] + n > H->c.max_ctx) return fail(H, DG_ECAPACITY, "prefill of %d exceeds max_ctx", n);
  if (n == 0) return DG_OK;
  return encode_causal(H, bi, tokens, n, n);
}

// where a step writes its argmax rows: the caller's buffer (the two-round stop requires one), else nowhere
static int32_t* argmax_target(const dg_step_out* o) { return (o && o->argmax) ? o->argmax : nullptr; }

int dg_sample(dg_handle* H, const float* logits, int batch, const int* req, int step, const dg_sampler_params* sp,
              int32_t* canvas, const dg_step_out* o) {
  if (!H) return DG_EINVAL;
  BatchInfo bi;
  int rc = make_batch(H, batch, req, &bi);
  if (rc) return rc;
  if ((rc = check_sampler_params(H, sp))) return rc;
  if (!logits || !canvas) return fail(H, DG_EINVAL, "null logits or canvas");
  if (!aligned16(logits)) return fail(H, DG_EINVAL, "logits must be 16-byte aligned");
  if (sp->stop_mode == DG_STOP_TWO_ROUNDS && !(o && o->argmax))
    return fail(H, DG_EINVAL, "the two-round stop needs o->argmax (the next round's prev_argmax)");
  if ((rc = upload_req(H, bi))) return rc;
  const SamplerArgs a = sampler_args(*sp, step);
  run_sampler(H, logits, bi, a, canvas, (o && o->x_hat) ? o->x_hat : H->xh[0], (o && o->pmax) ? o->pmax : H->pmax,
              (o && o->entropy) ? o->entropy : H->ent, o ? o->keep : nullptr, o ? o->mean_entropy : nullptr,
              o ? o->stop : nullptr, nullptr, nullptr, 0, argmax_target(o));
  return check_launch(H, "sample");
}

int dg_denoise_step(dg_handle* H, const dg_step_args* a, const dg_step_out* o) {
  if (!H || !a) return DG_EINVAL;
  const dg_config& c = H->c;
  if (c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  BatchInfo bi;
  int rc = make_batch(H, a->batch, a->req, &bi);
  if (rc) return rc;
  if ((rc = check_sampler_params(H, &a->sp))) return rc;
  if (!a->canvas) return fail(H, DG_EINVAL, "null canvas");
  if (a->logits_out && !aligned16(a->logits_out)) return fail(H, DG_EINVAL, "logits_out must be 16-byte aligned");
  if (a->step < 1) return fail(H, DG_EINVAL, "step must be >= 1");
  for (int b = 0; b < bi.B; ++b)
    if (bi.len[b] + c.canvas > c.max_ctx) return fail(H, DG_ECAPACITY, "cache + canvas exceeds max_ctx");
  if (a->dump && (a->dump->layer < 0 || a->dump->layer >= c.n_layers))
    return fail(H, DG_EINVAL, "dump layer %d out of [0, %d)", a->dump->layer, c.n_layers);
  if (a->sp.stop_mode == DG_STOP_TWO_ROUNDS && !(o && o->argmax))
    return fail(H, DG_EINVAL, "the two-round stop needs o->argmax (the next round's prev_argmax)");
  if ((rc = upload_req(H, bi))) return rc;
  const SamplerArgs sa = sampler_args(a->sp, a->step);
  // without a logits buffer from the caller, the LM head feeds the sampler directly (no logits written)
  const bool fused = H->vstats && !a->logits_out;
  float* logits = fused ? nullptr : (a->logits_out ? a->logits_out : H->logits);
  run_layers(H, bi, c.canvas, false, a->canvas, a->prev_pred, true, logits, a->hidden_out, a->dump,
             fused ? &sa : nullptr);
  run_sampler(H, logits, bi, sa, a->canvas, (o && o->x_hat) ? o->x_hat : H->xh[0],
              (o && o->pmax) ? o->pmax : H->pmax, (o && o->entropy) ? o->entropy : H->ent, o ? o->keep : nullptr,
              o ? o->mean_entropy : nullptr, o ? o->stop : nullptr, nullptr, nullptr, 0, argmax_target(o));
  if (o && o->experts_touched)
    cudaMemcpyAsync(o->experts_touched, H->touched, c.n_layers * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                    H->stream);
  return check_launch(H, "denoise step");
}

static int generate_block_impl(dg_handle* H, const dg_block_args* a, int32_t* out_dev, int* steps_used) {
  const dg_config& c = H->c;
  if (c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  BatchInfo bi;
  int rc = make_batch(H, a->batch, a->req, &bi);
  if (rc) return rc;
  if (a->max_steps < 1 || a->schedule_steps < 1) return fail(H, DG_EINVAL, "max_steps and schedule_steps must be >= 1");
  if (!(a->temperature >= 0.f) || !(a->logit_scale_growth > 0.f)) return fail(H, DG_EINVAL, "bad temperature / growth");
  if (a->anneal && !(a->temperature > 0.f && a->temperature_end > 0.f && std::isfinite(a->temperature) &&
                     std::isfinite(a->temperature_end)))
    return fail(H, DG_EINVAL, "an annealed temperature needs finite ends > 0");
  if (a->keep_mode != DG_KEEP_TOPK && a->keep_mode != DG_KEEP_ENTROPY_BUDGET)
    return fail(H, DG_EINVAL, "unknown keep_mode %d", a->keep_mode);
  if (a->keep_mode == DG_KEEP_ENTROPY_BUDGET && !(a->entropy_budget >= 0.f && std::isfinite(a->entropy_budget)))
    return fail(H, DG_EINVAL, "entropy_budget must be finite and >= 0");
  if (a->stop_mode != DG_STOP_MEAN_ENTROPY && a->stop_mode != DG_STOP_TWO_ROUNDS)
    return fail(H, DG_EINVAL, "unknown stop_mode %d", a->stop_mode);
  const bool two_rounds = a->stop_mode == DG_STOP_TWO_ROUNDS;
  for (int b = 0; b < bi.B; ++b)
    if (bi.len[b] + c.canvas > c.max_ctx) return fail(H, DG_ECAPACITY, "cache + canvas exceeds max_ctx");
  if ((rc = upload_req(H, bi))) return rc;
  const int n = c.canvas;
  {
    ProfScope ps(H, PC_FINISH);
    launch_init_canvas(H->canvas, bi, H->req_dev, n, c.vocab, a->seed, a->block, H->stream);
  }
  cudaMemsetAsync(H->done, 0, bi.B * sizeof(int32_t), H->stream);
  const int32_t* prev = nullptr;
  int steps = 0;
  for (int t = 1; t <= a->max_steps; ++t) {
    dg_sampler_params sp;
    sp.temperature = a->temperature;
    if (a->anneal) {
      // linear from T at step 1 to T_end at step max_steps, in double ([P1 四])
      const double t0 = a->temperature, t1 = a->temperature_end;
      sp.temperature = a->max_steps <= 1 ? a->temperature_end
                                         : (float)(t0 + (t1 - t0) * (double)(t - 1) / (double)(a->max_steps - 1));
    }
    sp.logit_scale = (float)std::pow((double)a->logit_scale_growth, (double)(t - 1));
    sp.stop_threshold = a->stop_threshold;
    sp.keep_k = std::min(n, (int)(((long long)n * t + a->schedule_steps - 1) / a->schedule_steps));
    sp.seed = a->seed;
    sp.block = a->block;
    sp.keep_mode = a->keep_mode;
    sp.entropy_budget = a->entropy_budget;
    // the two-round stop compares with the previous round's argmax and mean entropy (double-buffered)
    sp.stop_mode = a->stop_mode;
    sp.prev_argmax = (two_rounds && t > 1) ? H->amax[(t - 1) & 1] : nullptr;
    sp.prev_mean_entropy = (two_rounds && t > 1) ? H->mh2[(t - 1) & 1] : nullptr;
    if ((rc = check_sampler_params(H, &sp))) return rc;
    const SamplerArgs sa = sampler_args(sp, t);
    const bool fused = H->vstats != nullptr;
    run_layers(H, bi, n, false, H->canvas, prev, true, fused ? nullptr : H->logits, nullptr, nullptr,
               fused ? &sa : nullptr);
    int32_t* xh = H->xh[t & 1];
    run_sampler(H, fused ? nullptr : H->logits, bi, sa, H->canvas, xh, H->pmax, H->ent, H->keep,
                two_rounds ? H->mh2[t & 1] : H->meanh, H->stop, H->done, out_dev, t == a->max_steps ? 1 : 0,
                two_rounds ? H->amax[t & 1] : nullptr);
    if ((rc = check_launch(H, "block step"))) return rc;
    steps = t;
    cudaMemcpyAsync(H->h_done, H->done, bi.B * sizeof(int32_t), cudaMemcpyDeviceToHost, H->stream);
    if ((rc = cuda_check(H, cudaStreamSynchronize(H->stream), "block step sync"))) return rc;
    if ((rc = read_device_error(H))) return rc;
    bool all = true;
    for (int b = 0; b < bi.B; ++b) all &= H->h_done[b] != 0;
    if (all) break;
    prev = xh;
  }
  // causal hand-off of the finished block into the cache ([P2 架构基础], [P3])
  if ((rc = encode_causal(H, bi, out_dev, n, n))) return rc;
  if (steps_used) *steps_used = steps;
  return DG_OK;
}

int dg_generate_block(dg_handle* H, const dg_block_args* a, int32_t* out_tokens, int* steps_used) {
  if (!H || !a || !out_tokens) return H ? fail(H, DG_EINVAL, "null argument") : DG_EINVAL;
  return generate_block_impl(H, a, out_tokens, steps_used);
}

int dg_generate_block_host(dg_handle* H, const dg_block_args* a, int32_t* out_tokens_host, int* steps_used) {
  if (!H || !a || !out_tokens_host) return H ? fail(H, DG_EINVAL, "null argument") : DG_EINVAL;
  int rc = generate_block_impl(H, a, H->out_tok, steps_used);
  if (rc) return rc;
  rc = cuda_check(H,
                  cudaMemcpyAsync(out_tokens_host, H->out_tok, (size_t)a->batch * H->c.canvas * sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, H->stream),
                  "copy tokens to host");
  if (rc) return rc;
  return cuda_check(H, cudaStreamSynchronize(H->stream), "sync");
}

int dg_synchronize(dg_handle* H) {
  if (!H) return DG_EINVAL;
  int rc = cuda_check(H, cudaStreamSynchronize(H->stream), "synchronize");
  if (rc) return rc;
  return read_device_error(H);
}

uint64_t dg_launch_count(const dg_handle* H) { return H ? H->launches : 0; }

int dg_profile_enable(dg_handle* H, int mask) {
  if (!H) return DG_EINVAL;
  H->prof = mask != 0;
  H->prof_mask = (uint32_t)mask;
  return DG_OK;
}

int dg_profile_reset(dg_handle* H) {
  if (!H) return DG_EINVAL;
  cudaStreamSynchronize(H->stream);
  H->recs.clear();
  H->pool_used = 0;
  return DG_OK;
}

int dg_profile_read(dg_handle* H, dg_profile_entry* out, int max_entries, int* n_entries) {
  if (!H || !n_entries) return DG_EINVAL;
  int rc = cuda_check(H, cudaStreamSynchronize(H->stream), "profile sync");
  if (rc) return rc;
  double ms[PC_COUNT] = {0};
  int cnt[PC_COUNT] = {0};
  for (const auto& r : H->recs) {
    float t = 0.f;
    cudaEventElapsedTime(&t, r.a, r.b);
    ms[r.cls] += t;
    cnt[r.cls] += 1;
  }
  int n = 0;
  for (int k = 0; k < PC_COUNT; ++k) {
    if (cnt[k] == 0) continue;
    if (out && n < max_entries) {
      out[n].name = kProfNames[k];
      out[n].launches = cnt[k];
      out[n].ms = ms[k];
    }
    ++n;
  }
  *n_entries = n;
  return DG_OK;
}

int dg_selftest_philox(dg_handle* H, const uint32_t* ctr, const uint32_t* key, uint32_t* out, uint32_t* out_curand,
                       int n) {
  if (!H || !ctr || !key || !out || n < 0) return DG_EINVAL;
  launch_philox_selftest(ctr, key, out, out_curand, n, H->stream);
  H->launches += 1;
  return check_launch(H, "philox selftest");
}

int dg_selftest_gemm(dg_handle* H, const void* x, const void* w, int T, int M, int K, float* out) {
  if (!H || !x || !w || !out || T < 1 || M < 1 || K < 64 || K % 64) return H ? fail(H, DG_EINVAL, "bad gemm args") : DG_EINVAL;
  if (!aligned16(x) || !aligned16(w)) return fail(H, DG_EINVAL, "unaligned operands");
  TcGemm g{};
  g.mode = 0;
  g.M = M;
  g.K = K;
  g.T = T;
  g.ntile = pick_ntile((M + 127) / 128, T, H->num_sms);
  g.seg1 = g.seg2 = INT_MAX;
  g.epi = EPI_STORE_F32;
  g.out = out;
  g.ld_out = M;
  g.err = H->d_err;
  g.ksub = ksub_for(0, g.ntile);
  g.ctas_per_sm = ctas_for(g.ntile);
  CUtensorMap mx, mw;
  if (!tmap_chunks(&mx, x, K, T, K, (uint32_t)g.ntile, (uint32_t)g.ksub) ||
      !tmap_chunks(&mw, w, K, M, K, 128, (uint32_t)g.ksub))
    return fail(H, DG_ECUDA, "tensor map encode failed");
  CUtensorMap to;
  const bool tma_out = tmap_out3d(&to, out, M, T, 1, M);
  if (launch_gemm_tc(mw, mw, mw, mx, nullptr, g, H->num_sms, H->stream, tma_out ? &to : nullptr) != 0)
    return fail(H, DG_EINVAL, "GEMM tiling rejected");
  H->launches += 1;
  return check_launch(H, "selftest gemm");
}

int dg_selftest_gemm_split(dg_handle* H, const void* x, const void* w, int T, int M, int K, float* part,
                           int max_split, int* nsplit) {
  if (!H || !x || !w || !part || !nsplit || T < 1 || M < 1 || K < 64 || K % 64 || max_split < 1)
    return H ? fail(H, DG_EINVAL, "bad gemm args") : DG_EINVAL;
  if (!H->bf16) return fail(H, DG_ESTATE, "needs a bf16 handle");
  if (!aligned16(x) || !aligned16(w)) return fail(H, DG_EINVAL, "unaligned operands");
  const SplitPlan p = split_plan(H->num_sms, T, M, K, (size_t)max_split * T * M);
  if (p.split < 1) return fail(H, DG_EINVAL, "T = %d is above the split-K form's %d rows", T, kDenseSplitRows);
  CUtensorMap mx, mw;
  if (!tmap_chunks(&mx, x, K, T, K, (uint32_t)p.ntile, (uint32_t)p.ksub) ||
      !tmap_chunks(&mw, w, K, M, K, 128, (uint32_t)p.ksub))
    return fail(H, DG_ECUDA, "tensor map encode failed");
  run_split(H, mw, mw, mw, &mx, INT_MAX, INT_MAX, T, M, K, p, part);
  H->launches += 1;
  *nsplit = p.split;
  return check_launch(H, "selftest split gemm");
}

int dg_selftest_gemm_pair(dg_handle* H, const void* x, const void* w, int T, int M, int K, int ntile, int ksplit,
                          float* part) {
  if (!H || !x || !w || !part || T < 1 || M < 1 || K < 64 || K % 64 || ksplit < 1 || ksplit > K / 64 ||
      (ntile != 64 && ntile != 128 && ntile != 256))
    return H ? fail(H, DG_EINVAL, "bad pair gemm args") : DG_EINVAL;
  if (!H->bf16) return fail(H, DG_ESTATE, "needs a bf16 handle");
  if (!aligned16(x) || !aligned16(w)) return fail(H, DG_EINVAL, "unaligned operands");
  TcGemm g{};
  g.mode = 0;
  g.M = M;
  g.K = K;
  g.T = T;
  g.ntile = ntile;
  g.seg1 = g.seg2 = INT_MAX;
  g.epi = EPI_STORE_F32;
  g.out = part;
  g.ld_out = M;
  g.err = H->d_err;
  g.ksplit = ksplit;
  g.split_stride = (size_t)T * M;
  g.ksub = DG_PAIR_KSUB;
  while (g.ksub > 1 && ksplit > (K / 64 + g.ksub - 1) / g.ksub) g.ksub >>= 1;
  CUtensorMap mx, mw, to;
  if (!tmap_chunks(&mx, x, K, T, K, (uint32_t)(ntile / 2), (uint32_t)g.ksub) ||
      !tmap_chunks(&mw, w, K, M, K, 128, (uint32_t)g.ksub))
    return fail(H, DG_ECUDA, "tensor map encode failed");
  const bool tma_out = tmap_out3d(&to, part, M, T, ksplit, M);
  if (launch_gemm_tc_pair(mw, mw, mw, mx, g, H->num_sms, H->stream, tma_out ? &to : nullptr) != 0)
    return fail(H, DG_EINVAL, "pair GEMM tiling rejected");
  H->launches += 1;
  return check_launch(H, "selftest pair gemm");
}

int dg_ar_step(dg_handle* H, int batch, const int* req, const int32_t* tokens, float* logits, int32_t* next_token) {
  if (!H) return DG_EINVAL;
  const dg_config& c = H->c;
  if (c.n_layers == 0) return fail(H, DG_ESTATE, "sampler-only handle");
  BatchInfo bi;
  int rc = make_batch(H, batch, req, &bi);
  if (rc) return rc;
  if (!tokens || !logits) return fail(H, DG_EINVAL, "null tokens or logits");
  if (!aligned16(logits)) return fail(H, DG_EINVAL, "logits must be 16-byte aligned");
  for (int b = 0; b < bi.B; ++b)
    if (bi.len[b] + 1 > c.max_ctx) return fail(H, DG_ECAPACITY, "cache full: P + 1 exceeds max_ctx");
  if ((rc = upload_req(H, bi))) return rc;
  // causal encode of one token per request at position P, then the tied LM head on it
  run_layers(H, bi, 1, true, tokens, nullptr, true, logits, nullptr);
  if (next_token) {
    SamplerArgs a{};
    a.temperature = 0.f;   // argmax, ties to the lower index
    a.logit_scale = 1.f;
    a.stop_threshold = -1.f;
    ProfScope ps(H, PC_SAMPLER, 2);
    launch_sampler_rows(logits, bi.B, 1, c.vocab, H->req_dev, a, H->sws, next_token, H->pmax, H->ent, H->stream);
  }
  if ((rc = check_launch(H, "ar step"))) return rc;
  for (int b = 0; b < bi.B; ++b) H->len[bi.slot[b]] += 1;
  return DG_OK;
}

int dg_selftest_wait_timeout(dg_handle* H, int limit_us) {
  if (!H) return DG_EINVAL;
  if (limit_us < 1 || limit_us > 100000) return fail(H, DG_EINVAL, "limit_us out of [1, 100000]");
  int rc = cuda_check(H, cudaStreamSynchronize(H->stream), "wait self-test: drain");
  if (rc) return rc;
  if ((rc = read_device_error(H))) return rc;
  launch_wait_timeout_selftest(H->d_err, (unsigned long long)limit_us * 1000ull, H->stream);
  H->launches += 1;
  if ((rc = check_launch(H, "wait self-test"))) return rc;
  return dg_synchronize(H);
}

int dg_selftest_router(dg_handle* H, const float* logits, const float* bias, int T, int E, int k, int tile,
                       const dg_router_out* o) {
  if (!H) return DG_EINVAL;
  if (!logits || !o || !o->ids || !o->wts || !o->cnt || !o->off || !o->perm || !o->work || !o->n_work ||
      !o->touched)
    return fail(H, DG_EINVAL, "null router self-test argument");
  if (T < 1 || E < 1 || E > 256 || k < 1 || k > 16 || k > E || tile < 1 || tile > 1024)
    return fail(H, DG_EINVAL, "router self-test shape out of range (T %d, E %d, k %d, tile %d)", T, E, k, tile);
  if ((long long)T * k > (long long)INT_MAX / 2) return fail(H, DG_EINVAL, "T * k too large");
  launch_router_topk(logits, 1, bias, o->ids, o->wts, T, E, k, H->stream);
  launch_router_permute(o->ids, T * k, E, tile, o->cnt, o->off, o->perm, o->work, o->n_work, o->touched, H->stream);
  H->launches += 2;
  return check_launch(H, "router self-test");
}

}  // extern "C"
