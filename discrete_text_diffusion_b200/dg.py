"""Thin Python binding of the C ABI in include/dg.h (ctypes; argument
marshalling only).  Every function here forwards to the function of the same
name in libdg.so; tensors are passed as raw device pointers.

The library must have been built (``python -m discrete_text_diffusion_b200.build``);
importing this module without it raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DG_LIB selects another build of the library (default: the in-tree libdg.so)
LIB_PATH = os.environ.get("DG_LIB") or os.path.join(_HERE, "libdg.so")

DG_OK, DG_EINVAL, DG_ENOMEM, DG_ECUDA, DG_ECAPACITY, DG_ESTATE, DG_ETIMEOUT = range(7)
DG_FP32, DG_BF16 = 0, 1

EXPORTS = (
    "dg_create", "dg_destroy", "dg_last_error", "dg_prefill_prompt", "dg_set_kv", "dg_set_length",
    "dg_get_length", "dg_denoise_step", "dg_sample", "dg_generate_block", "dg_generate_block_host",
    "dg_synchronize", "dg_launch_count", "dg_profile_enable", "dg_profile_read", "dg_profile_reset",
    "dg_selftest_philox", "dg_selftest_gemm", "dg_sample_noalloc", "dg_selftest_gemm_split", "dg_selftest_gemm_pair", "dg_get_kv",
    "dg_selftest_router", "dg_selftest_wait_timeout", "dg_ar_step", "dg_quantize_nvfp4",
)


class DgConfig(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d_model", C.c_int), ("n_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int), ("d_ff", C.c_int),
                ("vocab", C.c_int), ("canvas", C.c_int), ("max_batch", C.c_int), ("max_ctx", C.c_int),
                ("max_tokens", C.c_int), ("dtype", C.c_int), ("rope_base", C.c_double), ("rms_eps", C.c_double),
                ("expert_format", C.c_int)]


class DgLayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "router_w",
                                          "router_b", "w_gate", "w_up", "w_down", "w_gate_sf", "w_up_sf",
                                          "w_down_sf", "w_gate_g", "w_up_g", "w_down_g")]


class DgWeights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("w_sc", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(DgLayerWeights))]


class DgSamplerParams(C.Structure):
    _fields_ = [("temperature", C.c_float), ("logit_scale", C.c_float), ("stop_threshold", C.c_float),
                ("keep_k", C.c_int), ("seed", C.c_uint64), ("block", C.c_uint32), ("keep_mode", C.c_int),
                ("entropy_budget", C.c_float), ("stop_mode", C.c_int), ("prev_argmax", C.c_void_p),
                ("prev_mean_entropy", C.c_void_p)]


DG_EXPERT_DTYPE = 0
DG_EXPERT_NVFP4 = 1

DG_KEEP_TOPK = 0
DG_KEEP_ENTROPY_BUDGET = 1
DG_STOP_MEAN_ENTROPY = 0
DG_STOP_TWO_ROUNDS = 1


class DgStepOut(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("x_hat", "pmax", "entropy", "keep", "mean_entropy", "stop",
                                          "experts_touched", "argmax")]


class DgLayerDump(C.Structure):
    _fields_ = [("layer", C.c_int), ("hidden_in", C.c_void_p), ("hidden_out", C.c_void_p),
                ("expert_ids", C.c_void_p), ("expert_wts", C.c_void_p)]


class DgStepArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("req", C.POINTER(C.c_int)), ("canvas", C.c_void_p),
                ("prev_pred", C.c_void_p), ("step", C.c_int), ("sp", DgSamplerParams),
                ("logits_out", C.c_void_p), ("hidden_out", C.c_void_p), ("dump", C.POINTER(DgLayerDump))]


class DgRouterOut(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("ids", "wts", "cnt", "off", "perm", "work", "n_work", "touched")]


class DgBlockArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("req", C.POINTER(C.c_int)), ("max_steps", C.c_int),
                ("schedule_steps", C.c_int), ("temperature", C.c_float), ("logit_scale_growth", C.c_float),
                ("stop_threshold", C.c_float), ("seed", C.c_uint64), ("block", C.c_uint32),
                ("keep_mode", C.c_int), ("entropy_budget", C.c_float), ("anneal", C.c_int),
                ("temperature_end", C.c_float), ("stop_mode", C.c_int)]


class DgProfileEntry(C.Structure):
    _fields_ = [("name", C.c_char_p), ("launches", C.c_int), ("ms", C.c_double)]


_lib = None


def lib():
    """Load libdg.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m discrete_text_diffusion_b200.build")
        L = C.CDLL(LIB_PATH)
        P = C.c_void_p
        L.dg_create.argtypes = [C.POINTER(DgConfig), C.POINTER(DgWeights), P, C.POINTER(P)]
        L.dg_destroy.argtypes = [P]
        L.dg_destroy.restype = None
        L.dg_last_error.argtypes = [P]
        L.dg_last_error.restype = C.c_char_p
        L.dg_prefill_prompt.argtypes = [P, C.c_int, C.POINTER(C.c_int), P, C.c_int]
        L.dg_set_kv.argtypes = [P, C.c_int, C.c_int, P, P, C.c_int]
        L.dg_get_kv.argtypes = [P, C.c_int, C.c_int, P, P, C.c_int]
        L.dg_selftest_router.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(DgRouterOut)]
        L.dg_selftest_wait_timeout.argtypes = [P, C.c_int]
        L.dg_ar_step.argtypes = [P, C.c_int, C.POINTER(C.c_int), P, P, P]
        L.dg_quantize_nvfp4.argtypes = [P, C.c_int, C.c_int, C.c_int, P, P, P, P, C.c_char_p, C.c_size_t]
        L.dg_set_length.argtypes = [P, C.c_int, C.c_int]
        L.dg_get_length.argtypes = [P, C.c_int, C.POINTER(C.c_int)]
        L.dg_denoise_step.argtypes = [P, C.POINTER(DgStepArgs), C.POINTER(DgStepOut)]
        L.dg_sample.argtypes = [P, P, C.c_int, C.POINTER(C.c_int), C.c_int, C.POINTER(DgSamplerParams), P,
                                C.POINTER(DgStepOut)]
        L.dg_generate_block.argtypes = [P, C.POINTER(DgBlockArgs), P, C.POINTER(C.c_int)]
        L.dg_generate_block_host.argtypes = [P, C.POINTER(DgBlockArgs), P, C.POINTER(C.c_int)]
        L.dg_synchronize.argtypes = [P]
        L.dg_launch_count.argtypes = [P]
        L.dg_launch_count.restype = C.c_uint64
        L.dg_profile_enable.argtypes = [P, C.c_int]
        L.dg_profile_read.argtypes = [P, C.POINTER(DgProfileEntry), C.c_int, C.POINTER(C.c_int)]
        L.dg_profile_reset.argtypes = [P]
        L.dg_selftest_philox.argtypes = [P, P, P, P, P, C.c_int]
        L.dg_selftest_gemm.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, P]
        L.dg_selftest_gemm_split.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, P, C.c_int, C.POINTER(C.c_int)]
        L.dg_selftest_gemm_pair.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P]
        L.dg_sample_noalloc.argtypes = [P, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_int), C.c_int,
                                        C.POINTER(DgSamplerParams), P, C.POINTER(DgStepOut), P, C.c_char_p,
                                        C.c_size_t]
        _lib = L
    return _lib


class DgError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"dg error {code}: {msg}")
        self.code = code


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _ints(xs):
    return (C.c_int * len(xs))(*[int(x) for x in xs])


class Handle:
    """Owns a dg_handle and keeps the borrowed weight tensors alive."""

    def __init__(self, ptr, keep):
        self.ptr = ptr
        self._keep = keep

    def check(self, rc):
        if rc != DG_OK:
            raise DgError(rc, lib().dg_last_error(self.ptr).decode())
        return rc

    def close(self):
        if self.ptr:
            lib().dg_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _cfg(model: dict, *, dtype: str, max_batch: int, max_ctx: int, max_tokens: int = 0,
         expert_format: int = DG_EXPERT_DTYPE) -> DgConfig:
    m = model
    return DgConfig(m.get("n_layers", 0), m.get("d_model", 0), m.get("n_heads", 0), m.get("n_kv_heads", 0),
                    m.get("head_dim", 0), m.get("n_experts", 0), m.get("top_k", 0), m.get("d_ff", 0),
                    m["vocab"], m["canvas"], max_batch, max_ctx, max_tokens,
                    DG_BF16 if dtype == "bf16" else DG_FP32, float(m.get("rope_base", 10000.0)),
                    float(m.get("rms_eps", 1e-6)), expert_format)


def dg_create(model: dict, weights, *, dtype: str, max_batch: int, max_ctx: int, max_tokens: int = 0,
              stream=None, expert_format: int = DG_EXPERT_DTYPE) -> Handle:
    """dg_create.  weights: dict of device tensors (synth.make_weights layout) or None
    for a sampler-only handle (model['n_layers'] == 0).  With expert_format
    DG_EXPERT_NVFP4 each layer's w_gate / w_up / w_down are the codes and the layer
    also holds w_gate_sf ... w_down_g (see dg_quantize_nvfp4)."""
    cfg = _cfg(model, dtype=dtype, max_batch=max_batch, max_ctx=max_ctx, max_tokens=max_tokens,
               expert_format=expert_format)
    keep = [weights]
    wp = None
    if weights is not None:
        lay = (DgLayerWeights * len(weights["layers"]))()
        for i, L in enumerate(weights["layers"]):
            for k in DgLayerWeights._fields_:
                name = k[0]
                setattr(lay[i], name, None if L.get(name) is None else L[name].data_ptr())
        keep.append(lay)
        wp = DgWeights(weights["embed"].data_ptr(), weights["w_sc"].data_ptr(), weights["final_norm"].data_ptr(),
                       lay)
        keep.append(wp)
    out = C.c_void_p()
    s = None if stream is None else C.c_void_p(stream.cuda_stream)
    rc = lib().dg_create(C.byref(cfg), C.byref(wp) if wp is not None else None, s, C.byref(out))
    if rc != DG_OK:
        raise DgError(rc, lib().dg_last_error(None).decode())
    return Handle(out, keep)


def dg_destroy(h: Handle):
    h.close()


def dg_last_error(h: Handle | None = None) -> str:
    return lib().dg_last_error(None if h is None else h.ptr).decode()


def dg_prefill_prompt(h: Handle, req, tokens: torch.Tensor):
    """tokens: int32 [B, n] on the device."""
    return h.check(lib().dg_prefill_prompt(h.ptr, len(req), _ints(req), _ptr(tokens), tokens.shape[-1]))


def dg_set_kv(h: Handle, req: int, layer: int, k: torch.Tensor, v: torch.Tensor):
    return h.check(lib().dg_set_kv(h.ptr, req, layer, _ptr(k), _ptr(v), k.shape[1]))


def dg_get_kv(h: Handle, req: int, layer: int, k: torch.Tensor, v: torch.Tensor):
    """Read positions [0, n) of a request's cache of one layer into k, v [Hkv, n, hd]."""
    return h.check(lib().dg_get_kv(h.ptr, req, layer, _ptr(k), _ptr(v), k.shape[1]))


def dg_set_length(h: Handle, req: int, length: int):
    return h.check(lib().dg_set_length(h.ptr, req, length))


def dg_get_length(h: Handle, req: int) -> int:
    v = C.c_int()
    h.check(lib().dg_get_length(h.ptr, req, C.byref(v)))
    return v.value


def sampler_params(temperature=1.0, logit_scale=1.0, stop_threshold=-1.0, keep_k=0, seed=0, block=0,
                   entropy_budget=None, two_round_stop=False, prev_argmax=None, prev_mean_entropy=None):
    """entropy_budget=None keeps the top keep_k by pmax; a number selects the entropy-budget keep.
    two_round_stop selects the stop on two rounds' mean entropies and argmax; prev_argmax [B, N] int32 and
    prev_mean_entropy [B] float32 (device tensors) are the previous round's outputs, None at the first round."""
    mode = DG_KEEP_TOPK if entropy_budget is None else DG_KEEP_ENTROPY_BUDGET
    return DgSamplerParams(temperature, logit_scale, stop_threshold, keep_k, seed, block, mode,
                           0.0 if entropy_budget is None else entropy_budget,
                           DG_STOP_TWO_ROUNDS if two_round_stop else DG_STOP_MEAN_ENTROPY,
                           None if prev_argmax is None else prev_argmax.data_ptr(),
                           None if prev_mean_entropy is None else prev_mean_entropy.data_ptr())


def step_out(x_hat=None, pmax=None, entropy=None, keep=None, mean_entropy=None, stop=None, experts_touched=None,
             argmax=None):
    return DgStepOut(*[None if t is None else t.data_ptr() for t in
                       (x_hat, pmax, entropy, keep, mean_entropy, stop, experts_touched, argmax)])


def layer_dump(layer, hidden_in=None, hidden_out=None, expert_ids=None, expert_wts=None):
    """A dg_layer_dump: record one layer of the next forward pass into these device tensors."""
    return DgLayerDump(layer, *[None if t is None else t.data_ptr()
                                for t in (hidden_in, hidden_out, expert_ids, expert_wts)])


def dg_denoise_step(h: Handle, req, canvas, prev_pred, step, sp: DgSamplerParams, out: DgStepOut,
                    logits_out=None, hidden_out=None, dump: DgLayerDump = None):
    a = DgStepArgs(len(req), _ints(req), canvas.data_ptr(), None if prev_pred is None else prev_pred.data_ptr(),
                   step, sp, None if logits_out is None else logits_out.data_ptr(),
                   None if hidden_out is None else hidden_out.data_ptr(),
                   None if dump is None else C.pointer(dump))
    return h.check(lib().dg_denoise_step(h.ptr, C.byref(a), C.byref(out)))


def dg_sample(h: Handle, logits, req, step, sp: DgSamplerParams, canvas, out: DgStepOut):
    return h.check(lib().dg_sample(h.ptr, _ptr(logits), len(req), _ints(req), step, C.byref(sp), _ptr(canvas),
                                   C.byref(out)))


def dg_sample_noalloc(logits, req, step, sp: DgSamplerParams, canvas, out: DgStepOut = None, stream=None):
    """dg_sample without a handle: logits [B, N, V] fp32 on the stream's device.
    stream: a torch.cuda.Stream (or None for the legacy default stream)."""
    B, n, V = logits.shape
    err = C.create_string_buffer(512)
    sptr = None if stream is None else C.c_void_p(stream.cuda_stream)
    rc = lib().dg_sample_noalloc(_ptr(logits), B, n, V, _ints(req), step, C.byref(sp), _ptr(canvas),
                                 None if out is None else C.byref(out), sptr, err, len(err))
    if rc != 0:
        raise DgError(rc, err.value.decode())
    return rc


def block_args(req, max_steps, schedule_steps, temperature=1.0, logit_scale_growth=1.0, stop_threshold=-1.0,
               seed=0, block=0, entropy_budget=None, temperature_end=None, two_round_stop=False):
    """entropy_budget: None = the k_t schedule, else the entropy-budget keep.
    temperature_end: None = constant temperature, else the linear anneal to it.
    two_round_stop: stop on two rounds' mean entropies (< stop_threshold) and an unchanged argmax."""
    mode = DG_KEEP_TOPK if entropy_budget is None else DG_KEEP_ENTROPY_BUDGET
    return DgBlockArgs(len(req), _ints(req), max_steps, schedule_steps, temperature, logit_scale_growth,
                       stop_threshold, seed, block, mode, 0.0 if entropy_budget is None else entropy_budget,
                       0 if temperature_end is None else 1, 0.0 if temperature_end is None else temperature_end,
                       DG_STOP_TWO_ROUNDS if two_round_stop else DG_STOP_MEAN_ENTROPY)


def dg_generate_block(h: Handle, a: DgBlockArgs, out_tokens: torch.Tensor) -> int:
    steps = C.c_int()
    h.check(lib().dg_generate_block(h.ptr, C.byref(a), _ptr(out_tokens), C.byref(steps)))
    return steps.value


def dg_generate_block_host(h: Handle, a: DgBlockArgs, out_tokens_host: torch.Tensor) -> int:
    steps = C.c_int()
    h.check(lib().dg_generate_block_host(h.ptr, C.byref(a), _ptr(out_tokens_host), C.byref(steps)))
    return steps.value


def dg_ar_step(h: Handle, req, tokens, logits, next_token=None):
    """AR mode: append tokens [B] (int32, device) causally; logits [B, V] fp32 of the next token;
    next_token [B] int32 (argmax) or None."""
    return h.check(lib().dg_ar_step(h.ptr, len(req), _ints(req), _ptr(tokens), _ptr(logits), _ptr(next_token)))


def nvfp4_scales_shape(n_mats: int, rows: int, K: int):
    """Shape of the tiled block scales dg_quantize_nvfp4 writes: [n_mats, K/64, rows_pad, 4]."""
    return (n_mats, K // 64, (rows + 127) // 128 * 128, 4)


def dg_quantize_nvfp4(w, codes, scales, g, stream=None):
    """w [n_mats, rows, K] bf16 -> codes [n_mats, rows, K/2] uint8, scales (nvfp4_scales_shape) uint8,
    g [n_mats] float32, all on the device."""
    n_mats, rows, K = w.shape
    err = C.create_string_buffer(256)
    sptr = None if stream is None else C.c_void_p(stream.cuda_stream)
    rc = lib().dg_quantize_nvfp4(_ptr(w), n_mats, rows, K, _ptr(codes), _ptr(scales), _ptr(g), sptr, err, len(err))
    if rc != 0:
        raise DgError(rc, err.value.decode())
    return rc


def dg_synchronize(h: Handle):
    return h.check(lib().dg_synchronize(h.ptr))


def dg_launch_count(h: Handle) -> int:
    return int(lib().dg_launch_count(h.ptr))


# profiler kernel classes in the header's order (bit k of the mask = class k)
PROFILE_CLASSES = ("embed", "dense_gemm", "rope_scatter", "attention", "rmsnorm", "router", "gather", "moe_up",
                   "moe_down", "combine", "lm_head", "sampler_rows", "sampler_finish")


def dg_profile_enable(h: Handle, on: bool, classes=None):
    """on=False: off; on=True: every class, or only the named ``classes``."""
    mask = 0
    if on:
        mask = -1 if classes is None else sum(1 << PROFILE_CLASSES.index(c) for c in classes)
    return h.check(lib().dg_profile_enable(h.ptr, mask))


def dg_profile_reset(h: Handle):
    return h.check(lib().dg_profile_reset(h.ptr))


def dg_profile_read(h: Handle) -> dict:
    arr = (DgProfileEntry * 32)()
    n = C.c_int()
    h.check(lib().dg_profile_read(h.ptr, arr, 32, C.byref(n)))
    return {arr[i].name.decode(): (arr[i].launches, arr[i].ms) for i in range(min(n.value, 32))}


def dg_selftest_philox(h: Handle, ctr, key, out, out_curand=None):
    return h.check(lib().dg_selftest_philox(h.ptr, _ptr(ctr), _ptr(key), _ptr(out), _ptr(out_curand),
                                            ctr.shape[0]))


def dg_selftest_gemm(h: Handle, x, w, out):
    """out[T, M] fp32 = x[T, K] @ w[M, K]^T through the tensor-core GEMM."""
    return h.check(lib().dg_selftest_gemm(h.ptr, _ptr(x), _ptr(w), x.shape[0], w.shape[0], x.shape[1], _ptr(out)))


def dg_selftest_wait_timeout(h: Handle, limit_us: int) -> int:
    """Run the wait self-test; returns the status code (DG_ETIMEOUT when the wait gave up as designed)."""
    return int(lib().dg_selftest_wait_timeout(h.ptr, int(limit_us)))


def dg_selftest_router(h: Handle, logits, bias, k: int, tile: int, out: dict):
    """Router self-test on logits [T, E] fp32 (+ bias [E] or None); out: dict of device tensors
    ids, wts, cnt, off, perm, work, n_work, touched."""
    T, E = logits.shape
    o = DgRouterOut(*[out[n].data_ptr() for n, _ in DgRouterOut._fields_])
    return h.check(lib().dg_selftest_router(h.ptr, _ptr(logits), _ptr(bias), T, E, k, tile, C.byref(o)))


def dg_selftest_gemm_pair(h: Handle, x, w, part, ntile):
    """x @ w.T on CTA pairs as part.shape[0] split-K fp32 slices part [ksplit, T, M]."""
    return h.check(lib().dg_selftest_gemm_pair(h.ptr, _ptr(x), _ptr(w), x.shape[0], w.shape[0], x.shape[1], ntile,
                                               part.shape[0], _ptr(part)))


def dg_selftest_gemm_split(h: Handle, x, w, part):
    """Split-K partial slices of x @ w.T into part [max_split, T, M]; returns the slice count."""
    n = C.c_int()
    h.check(lib().dg_selftest_gemm_split(h.ptr, _ptr(x), _ptr(w), x.shape[0], w.shape[0], x.shape[1], _ptr(part),
                                         part.shape[0], C.byref(n)))
    return n.value
