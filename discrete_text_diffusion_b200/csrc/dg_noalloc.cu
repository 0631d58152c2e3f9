// dg_sample_noalloc: the sampler (same kernels and results as dg_sample) for
// callers that may not allocate device memory and hold no handle.
//
// Who needs it: code that runs inside a memory-planned runtime (a serving
// engine that reserved all HBM up front, a caching allocator it must not
// bypass), or that samples from logits it already owns without creating a
// handle, whose dg_create would cudaMalloc the KV cache and workspaces.
// Neither cudaMalloc nor cudaFree nor any allocating library routine is
// called here: the per-call scratch (the sampler's per-chunk partial sums,
// the request ids, and x_hat / pmax / entropy when the caller does not want
// them) lives in one fixed file-scope device array, allocated once per device
// by the CUDA runtime when this library's module is loaded.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dg.h"
#include "dg_common.cuh"
#include "kernels.h"

using namespace dg;

namespace {

// The request ids travel as a kernel argument, so a call makes no host-to-device copy.
struct ReqIds {
  int32_t v[64];
};

__global__ void store_req_ids_kernel(ReqIds ids, int n, int32_t* dst) {
  pdl_wait();
  pdl_trigger();
  if ((int)threadIdx.x < n) dst[threadIdx.x] = ids.v[threadIdx.x];
}

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxReq = 64;                          // request ids held in the scratch
constexpr int kMaxDevices = 64;

// The scratch.  No byte of it has to start at zero: everything a call reads
// from it was written earlier in the same call.
__device__ __align__(256) unsigned char g_sample_scratch[kScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

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

int dg_sample_noalloc(const float* logits, int batch, int n, int vocab, const int* req, int step,
                      const dg_sampler_params* sp, int32_t* canvas, const dg_step_out* o, void* stream, char* err,
                      size_t err_len) {
  if (err && err_len > 0) err[0] = '\0';
  if (!logits || !canvas || !req || !sp) return report(err, err_len, DG_EINVAL, "null logits, canvas, req or params");
  if (((uintptr_t)logits & 15u) != 0) return report(err, err_len, DG_EINVAL, "logits must be 16-byte aligned");
  if (batch < 1 || batch > kMaxReq) return report(err, err_len, DG_EINVAL, "batch %d out of [1, %d]", batch, kMaxReq);
  if (n < 1 || n > 1024) return report(err, err_len, DG_EINVAL, "canvas length %d out of [1, 1024]", n);
  if (vocab < 1) return report(err, err_len, DG_EINVAL, "vocab must be >= 1");
  for (int b = 0; b < batch; ++b)
    if (req[b] < 0) return report(err, err_len, DG_EINVAL, "request id %d is negative", req[b]);
  if (!(sp->temperature >= 0.f) || !std::isfinite(sp->temperature))
    return report(err, err_len, DG_EINVAL, "temperature must be finite and >= 0");
  if (!(sp->logit_scale > 0.f) || !std::isfinite(sp->logit_scale))
    return report(err, err_len, DG_EINVAL, "logit_scale must be > 0");
  if (sp->keep_k < 0 || sp->keep_k > n) return report(err, err_len, DG_EINVAL, "keep_k out of [0, N]");
  if (sp->keep_mode != DG_KEEP_TOPK && sp->keep_mode != DG_KEEP_ENTROPY_BUDGET)
    return report(err, err_len, DG_EINVAL, "unknown keep_mode %d", sp->keep_mode);
  if (sp->keep_mode == DG_KEEP_ENTROPY_BUDGET && !(sp->entropy_budget >= 0.f && std::isfinite(sp->entropy_budget)))
    return report(err, err_len, DG_EINVAL, "entropy_budget must be finite and >= 0");
  if (sp->stop_mode != DG_STOP_MEAN_ENTROPY && sp->stop_mode != DG_STOP_TWO_ROUNDS)
    return report(err, err_len, DG_EINVAL, "unknown stop_mode %d", sp->stop_mode);
  if (sp->stop_mode == DG_STOP_TWO_ROUNDS && !(o && o->argmax))
    return report(err, err_len, DG_EINVAL, "the two-round stop needs o->argmax (the next round's prev_argmax)");

  // scratch layout: request ids | x_hat | pmax | entropy | chunk partials
  const size_t rows = (size_t)batch * n;
  const size_t off_xh = round256(kMaxReq * sizeof(int32_t));
  const size_t off_pm = off_xh + round256(rows * sizeof(int32_t));
  const size_t off_en = off_pm + round256(rows * sizeof(float));
  const size_t off_ws = off_en + round256(rows * sizeof(float));
  const size_t need = off_ws + round256(sampler_workspace_bytes((int)rows, vocab));
  if (need > kScratchBytes)
    return report(err, err_len, DG_ECAPACITY,
                  "batch %d x canvas %d x vocab %d needs %zu bytes of scratch; the fixed scratch holds %zu", batch, n,
                  vocab, need, kScratchBytes);

  // once per device, with that device current: the address of its copy of the scratch
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return report(err, err_len, DG_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return report(err, err_len, DG_EINVAL, "device ordinal %d unsupported", dev);
  unsigned char* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_sample_scratch);
      if (e != cudaSuccess || !p)
        return report(err, err_len, DG_ECUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      g_scratch_ptr[dev] = p;
    }
    base = static_cast<unsigned char*>(g_scratch_ptr[dev]);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* req_dev = reinterpret_cast<int32_t*>(base);
  ReqIds ids{};
  for (int b = 0; b < batch; ++b) ids.v[b] = req[b];
  e = launch_k(store_req_ids_kernel, dim3(1), dim3(kMaxReq), 0, s, ids, batch, req_dev);
  if (e != cudaSuccess) return report(err, err_len, DG_ECUDA, "request id store: %s", cudaGetErrorString(e));

  int32_t* xh = (o && o->x_hat) ? o->x_hat : reinterpret_cast<int32_t*>(base + off_xh);
  float* pmax = (o && o->pmax) ? o->pmax : reinterpret_cast<float*>(base + off_pm);
  float* ent = (o && o->entropy) ? o->entropy : reinterpret_cast<float*>(base + off_en);
  SamplerArgs a;
  a.temperature = sp->temperature;
  a.logit_scale = sp->logit_scale;
  a.stop_threshold = sp->stop_threshold;
  a.keep_k = sp->keep_k;
  a.seed = sp->seed;
  a.block = sp->block;
  a.step = (uint32_t)step;
  a.keep_mode = sp->keep_mode;
  a.entropy_budget = sp->entropy_budget;
  a.stop_mode = sp->stop_mode;
  a.prev_argmax = sp->prev_argmax;
  a.prev_mean_h = sp->prev_mean_entropy;
  int32_t* amax = (o && o->argmax) ? o->argmax : nullptr;
  launch_sampler_rows(logits, (int)rows, n, vocab, req_dev, a, base + off_ws, xh, pmax, ent, s, amax);
  launch_sampler_finish(xh, pmax, ent, batch, n, vocab, req_dev, a, canvas, o ? o->keep : nullptr,
                        o ? o->mean_entropy : nullptr, o ? o->stop : nullptr, nullptr, nullptr, 0, s, amax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return report(err, err_len, DG_ECUDA, "sampler launch: %s", cudaGetErrorString(e));
  return DG_OK;
}
