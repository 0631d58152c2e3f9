"""ctypes wrapper of the C++ oracle (TEST INFRASTRUCTURE).

Builds ``oracle/libdgoracle.so`` from ``oracle/dg_oracle.cpp`` with g++ on first
use (``build()``) and exposes its functions with numpy arguments.  Like the
numpy oracle, only ``tests/``, ``__graft_entry__`` and the bench's CPU-baseline
legs may use it; the CUDA library shares no code with it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dg_oracle.cpp")
LIB = os.path.join(HERE, "libdgoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (plain g++, OpenMP over independent rows, no fast-math,
    no floating-point contraction) unless the library is newer than its source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", SRC, "-o", LIB]
    subprocess.run(cmd, check=True)
    return LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        _lib.dgo_philox.argtypes = [P, P, P]
        _lib.dgo_init_canvas.argtypes = [C.c_uint64, C.c_int, C.c_uint32, C.c_uint32, C.c_uint32, P]
        _lib.dgo_layer.argtypes = ([C.c_int] * 7 + [C.c_double] * 2 + [P] * 11 +
                                   [P, C.c_int, P, P, P, C.c_int, C.c_int, P, P, C.c_int])
        _lib.dgo_router_select.argtypes = [P, C.c_int, C.c_int, C.c_int, P, P]
        _lib.dgo_embed.argtypes = [P, P, C.c_int, P, P, C.c_int, P]
        _lib.dgo_head.argtypes = [P, P, P, C.c_int, C.c_int, C.c_int, C.c_double, P]
        _lib.dgo_sample_canvas.argtypes = ([P, C.c_int, C.c_int, C.c_uint64, C.c_uint32, C.c_uint32, C.c_uint32,
                                            C.c_double, C.c_double, C.c_int, C.c_double] + [P] * 8)
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _p(a):
    """Address of a numpy array.  The caller keeps the array referenced until the call returns."""
    return None if a is None else C.c_void_p(a.ctypes.data)


def philox(ctr, key):
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().dgo_philox(_p(c), _p(k), _p(out))
    return out


def init_canvas(seed, n, vocab, block, req):
    out = np.zeros(n, dtype=np.int64)
    lib().dgo_init_canvas(int(seed), n, vocab, block, req, _p(out))
    return out


def router_select(g, top_k):
    g = _f64(g)
    T, E = g.shape
    ids = np.zeros((T, top_k), dtype=np.int64)
    w = np.zeros((T, top_k))
    lib().dgo_router_select(_p(g), T, E, top_k, _p(ids), _p(w))
    return ids, w


def layer(cfg, L, h, pos, k_cache, v_cache, causal, fp32=False):
    """One layer (the numpy oracle's OracleModel.layer): returns (h_out, k_new, v_new)."""
    hq, hkv, hd = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    h = _f64(h).copy()
    n = h.shape[0]
    kc, vc = _f64(k_cache), _f64(v_cache)
    P = kc.shape[1]
    k_new = np.zeros((hkv, n, hd))
    v_new = np.zeros((hkv, n, hd))
    w = {k: _f64(L[k]) for k in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "router_w", "w_gate", "w_up",
                                 "w_down")}
    rb = None if L.get("router_b") is None else _f64(L["router_b"])
    pos64 = _i64(pos)
    lib().dgo_layer(cfg["d_model"], hq, hkv, hd, cfg["n_experts"], cfg["top_k"], cfg["d_ff"], cfg["rope_base"],
                    cfg["rms_eps"], _p(w["attn_norm"]), _p(w["wq"]), _p(w["wk"]), _p(w["wv"]), _p(w["wo"]),
                    _p(w["ffn_norm"]), _p(w["router_w"]), _p(rb), _p(w["w_gate"]), _p(w["w_up"]), _p(w["w_down"]),
                    _p(h), n, _p(pos64), _p(kc), _p(vc), P, 1 if causal else 0, _p(k_new), _p(v_new),
                    1 if fp32 else 0)
    return h, k_new, v_new


def embed(E, w_sc, tokens, prev=None):
    E, w_sc, tok = _f64(E), _f64(w_sc), _i64(tokens)
    prv = None if prev is None else _i64(prev)
    n, d = len(tok), E.shape[1]
    h = np.zeros((n, d))
    lib().dgo_embed(_p(E), _p(w_sc), d, _p(tok), _p(prv), n, _p(h))
    return h


def head(h, final_norm, E, eps):
    h, E, fn = _f64(h), _f64(E), _f64(final_norm)
    n, d = h.shape
    out = np.zeros((n, E.shape[0]))
    lib().dgo_head(_p(h), _p(fn), _p(E), n, d, E.shape[0], eps, _p(out))
    return out


def sample_canvas(logits, *, seed, step, block, req, temperature, logit_scale, keep_k, stop_threshold):
    """The numpy oracle's sample_canvas (without the margins)."""
    lg = _f64(logits)
    N, V = lg.shape
    o = dict(x_hat=np.zeros(N, np.int64), pmax=np.zeros(N), H=np.zeros(N), keep=np.zeros(N, np.int32),
             x_new=np.zeros(N, np.int64), mean_H=np.zeros(1), stop=np.zeros(1, np.int32),
             argmax=np.zeros(N, np.int64))
    lib().dgo_sample_canvas(_p(lg), N, V, int(seed), step, block, req, float(temperature), float(logit_scale),
                            keep_k, float(stop_threshold), _p(o["x_hat"]), _p(o["pmax"]), _p(o["H"]), _p(o["keep"]),
                            _p(o["x_new"]), _p(o["mean_H"]), _p(o["stop"]), _p(o["argmax"]))
    o["keep"] = o["keep"].astype(bool)
    o["mean_H"] = float(o["mean_H"][0])
    o["stop"] = bool(o["stop"][0])
    return o


def denoise_forward(cfg, weights, caches, canvas, prev_pred=None, fp32=False):
    """A canvas forward pass through the C++ pieces: embed + self-conditioning,
    every layer (bidirectional, over the request's cache), final norm, tied LM
    head.  caches: per layer (k [Hkv, P, hd], v).  Returns logits [N, V]."""
    P = caches[0][0].shape[1]
    pos = P + np.arange(len(canvas))
    h = embed(weights["embed"], weights["w_sc"], canvas, prev_pred)
    for li, L in enumerate(weights["layers"]):
        h, _, _ = layer(cfg, L, h, pos, caches[li][0], caches[li][1], causal=False, fp32=fp32)
    return head(h, weights["final_norm"], weights["embed"], cfg["rms_eps"])
