"""Plain CPU oracle of the DiffusionGemma-style denoising step (TEST INFRASTRUCTURE).

This module is test infrastructure, not product code.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The CUDA library shares no code with it.

Everything is float64 numpy.  bf16 / fp32 inputs are upcast exactly.  Matrix
products use ``numpy.matmul`` as a library primitive; there is no blocking,
fusion or reordering beyond the definitions written out below.

Sources, cited by tag in the docstrings:
  [P1] "DiffusionGemma" technical-report summary (animattoys.com), sections
       一 (multinomial diffusion, canvas of 256 random tokens, ~12 rounds),
       二 (Gemma-4 MoE 128 experts / top-8, causal prompt + bidirectional canvas,
       self-conditioning, ~7.8M extra parameters),
       四 (the sampler: confidence, entropy, re-randomisation, temperature,
       adaptive stop), 五 (per-step cost: MoE, 262k-vocab softmax, attention).
  [P2] DiffusionGemma overview (youleyou.com), "架构基础" (causal encoder into the
       KV cache, bidirectional denoiser over the 256-token canvas, block-
       autoregressive hand-off) and "离散文本扩散的运作机制" (canvas init,
       iterative refinement, re-noising).
  [P3] "Google 開源 DiffusionGemma" (akiraxclaw.com blog): a finished canvas is
       encoded into the KV cache before the next canvas.
  [Philox] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
       1, 2, 3", SC'11: Philox4x32 with 10 rounds.

Readings of points the pages leave open (each is a named reading, R-x):
  R-noise   re-noise draws uniformly over the whole vocabulary [0, V) ([P1 一]).
  R-sample  multinomial draw by inverse CDF in vocabulary order with one Philox
            uniform per position; T == 0 means argmax (ties -> lower index).
  R-keep    keep the top-k positions by max-probability (ties -> lower index),
            re-selected every step; others are re-noised ([P1 四]: locked tokens
            can still change).
  R-stats   all statistics use z = s * l / T; entropy in nats; the stop test
            uses this step's statistics, before re-noise.
  R-sc      self-conditioning adds E[x_prev] @ W_sc^T to the token embedding;
            x_prev = previous step's sampled tokens; zero at the first step.
  R-norm    RMSNorm x * w / sqrt(mean(x^2) + eps).
  R-rope    rotate-half RoPE, pairs (j, j + hd/2), theta_j = base^(-2j/hd).
  R-router  logits + per-expert bias, top-k with ties to the lower id,
            softmax over the k selected logits.
  R-append  a finished canvas is appended by one causal encode pass over its
            tokens (no self-conditioning).
  R-ar      AR mode ([P1 七]: the weights load unchanged as an autoregressive
            model): a token is encoded causally at the end of the cache, as a
            prompt token is, and the tied LM head of its final-norm output
            gives the next token's logits.  No canvas, no self-conditioning.
  The page's own sampler variants ([P1 四]; the CUDA path has all three):
  R-budget  entropy-ordered locking: positions sorted by entropy ascending
            (ties -> lower index) are kept while the inclusive cumulative
            entropy stays <= the budget (0.1); the position that crosses it and
            all after it are re-noised.  Locking starts from the most certain
            position, so that one is kept whatever its entropy.
  R-anneal  the temperature falls linearly from 0.8 at round 1 to 0.4 at the
            last round of the step budget.
  R-stop2   stop after round t when the mean entropy of rounds t-1 and t is
            below 0.005 and the argmax sequence of round t equals round t-1's.

Parity pins: every public function here is pinned by ``tests/test_oracle_*.py``
against library routines, closed forms, invariants or brute force.  Parity
unpinned: none.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------
# Philox4x32-10 [Philox]: a 10-round bijection of a 128-bit counter under a
# 64-bit key.  One round multiplies words 0 and 2 by two constants, swaps the
# high/low halves across the pairs and xors in the key; the key is bumped by
# two Weyl constants between rounds.
# ----------------------------------------------------------------------------
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32-10 block function [Philox].

    ctr: uint32-compatible array [..., 4]; key: uint32-compatible array [..., 2]
    (broadcast against ctr).  Returns uint32 [..., 4].
    """
    ctr = np.asarray(ctr, dtype=np.uint64) & _MASK32
    key = np.asarray(key, dtype=np.uint64) & _MASK32
    c0, c1, c2, c3 = (ctr[..., i] for i in range(4))
    k0, k1 = key[..., 0], key[..., 1]
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c0          # < 2^64: exact in uint64
        p1 = _PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack(np.broadcast_arrays(c0, c1, c2, c3), axis=-1).astype(np.uint32)


def seed_key(seed: int):
    """64-bit seed -> Philox key (low word, high word)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint64)


def sampler_words(seed: int, pos, step: int, block: int, req: int):
    """The four Philox words of counter (position, step, block, request)."""
    pos = np.asarray(pos, dtype=np.uint64)
    ctr = np.stack(np.broadcast_arrays(pos, np.uint64(step), np.uint64(block),
                                       np.uint64(req)), axis=-1)
    return philox4x32_10(ctr, seed_key(seed))


def unit_uniform(w0):
    """u = (w0 >> 8) * 2^-24, in [0, 1) with 24 random bits (R-sample)."""
    return (np.asarray(w0, dtype=np.uint64) >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


def uniform_token(w1, vocab: int):
    """floor(w1 * V / 2^32): a token uniform over [0, V) (R-noise)."""
    return ((np.asarray(w1, dtype=np.uint64) * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)


def init_canvas(seed: int, n: int, vocab: int, block: int, req: int):
    """Canvas initialisation: n uniform-random vocabulary tokens ([P1 一], [P2]),
    drawn from word 1 of counter (i, 0, block, req)."""
    w = sampler_words(seed, np.arange(n), 0, block, req)
    return uniform_token(w[:, 1], vocab)


# ----------------------------------------------------------------------------
# Model pieces ([P1 二], [P2 架构基础]).
# ----------------------------------------------------------------------------

def rms_norm(x, w, eps):
    """R-norm: x * w / sqrt(mean(x^2) + eps) over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def rope(x, pos, base):
    """R-rope on x [..., n, hd] at integer positions pos [n]."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    theta = base ** (-2.0 * np.arange(half) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q, k, v, allowed=None):
    """Softmax attention with GQA head sharing.

    q [Hq, nq, hd]; k, v [Hkv, nk, hd]; allowed: bool [nq, nk] or None (no mask).
    Query head h reads KV head floor(h * Hkv / Hq); scores are scaled by
    1/sqrt(hd).  Returns [Hq, nq, hd].
    """
    hq, _, hd = q.shape
    hkv = k.shape[0]
    out = np.empty_like(q, dtype=np.float64)
    for h in range(hq):
        g = (h * hkv) // hq
        s = (q[h] @ k[g].T) / math.sqrt(hd)
        if allowed is not None:
            s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=-1, keepdims=True)
        out[h] = p @ v[g]
    return out


def silu(x):
    return x / (1.0 + np.exp(-x))


def swiglu_expert(x, w_gate, w_up, w_down):
    """One expert FFN: (silu(x Wg^T) * (x Wu^T)) Wd^T; W are [out, in]."""
    return (silu(x @ w_gate.T) * (x @ w_up.T)) @ w_down.T


def router(x, w_router, b_router, top_k):
    """R-router.  Returns (ids [T,k], weights [T,k], logits [T,E], margin [T]).

    margin = gap between the k-th and (k+1)-th largest logit (inf when k == E):
    the distance that decides the expert set.
    """
    g = x @ w_router.T
    if b_router is not None:
        g = g + np.asarray(b_router, np.float64)
    ids, w, margin = router_select(g, top_k)
    return ids, w, g, margin


def router_select(g, top_k):
    """The selection step of R-router on gate logits g [T, E] (bias included):
    the top_k experts by logit, ties to the lower id (-inf logits rank last,
    among themselves by id), and the softmax over the selected logits.
    Returns (ids [T,k] in selection order, weights [T,k], margin [T])."""
    g = np.asarray(g, np.float64)
    n_e = g.shape[1]
    idx = np.arange(n_e)
    ids = np.empty((g.shape[0], top_k), dtype=np.int64)
    margin = np.full(g.shape[0], np.inf)
    for t in range(g.shape[0]):
        order = np.lexsort((idx, -g[t]))          # logit descending, then id ascending
        ids[t] = order[:top_k]
        if top_k < n_e:
            a, b = g[t, order[top_k - 1]], g[t, order[top_k]]
            margin[t] = 0.0 if a == b else a - b          # -inf next to -inf is an exact tie
    sel = np.take_along_axis(g, ids, axis=1)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = e / e.sum(axis=1, keepdims=True)
    return ids, w, margin


def expert_order(ids, n_experts, tile):
    """The routed (token, slot) items grouped by expert, as the experts process
    them ([P1 二]: each token goes to its top-k experts of 128).  Item t*k+s is
    token t's s-th choice ids[t, s].

    Returns cnt [E] (items per expert), off [E+1] (exclusive prefix sum of cnt),
    perm [T*k] (the items of expert 0, then expert 1, ...; inside an expert by
    ascending item index, so tokens ascending), the work tiles [(expert, first
    position in perm, rows)] that cut each expert's run into pieces of at most
    `tile` rows (experts ascending), and the number of experts touched.
    """
    items = np.asarray(ids).reshape(-1)
    cnt = np.array([int(np.sum(items == e)) for e in range(n_experts)], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
    perm = np.empty(items.shape[0], dtype=np.int64)
    for e in range(n_experts):
        perm[off[e]:off[e + 1]] = np.nonzero(items == e)[0]
    work = [(e, int(off[e]) + r0, int(min(tile, cnt[e] - r0)))
            for e in range(n_experts) for r0 in range(0, int(cnt[e]), tile)]
    return cnt, off, perm, work, int(np.sum(cnt > 0))


def moe(x, layer, top_k):
    """Top-k mixture of SwiGLU experts ([P1 二]: 128 experts, 8 per token)."""
    ids, w, _, _ = router(x, layer["router_w"], layer.get("router_b"), top_k)
    out = np.zeros_like(x, dtype=np.float64)
    for e in np.unique(ids):
        tok, slot = np.nonzero(ids == e)
        y = swiglu_expert(x[tok], layer["w_gate"][e], layer["w_up"][e], layer["w_down"][e])
        out[tok] += w[tok, slot][:, None] * y
    return out


# ----------------------------------------------------------------------------
# Sampler ([P1 四], [P1 五]).
# ----------------------------------------------------------------------------

def position_stats(logits_row, temperature, logit_scale):
    """Per-position statistics of the tempered distribution (R-stats).

    Returns dict(z, e, S, pmax, H) with e = exp(z - max z), S = sum(e).
    T == 0 is the T -> 0+ limit: the uniform distribution over the maximal
    logits, so pmax = 1/c and H = log c for c tied maxima.
    """
    l = np.asarray(logits_row, dtype=np.float64) * float(logit_scale)
    if temperature == 0.0:
        c = int(np.count_nonzero(l == l.max()))
        return dict(z=l, e=None, S=float(c), pmax=1.0 / c, H=math.log(c))
    z = l / float(temperature)
    e = np.exp(z - z.max())
    S = float(e.sum())
    H = math.log(S) - float(np.dot(e, z - z.max())) / S
    return dict(z=z, e=e, S=S, pmax=1.0 / S, H=H)


def inverse_cdf(e, S, u):
    """Smallest j with sum_{i<=j} e_i > u*S (R-sample).  If rounding leaves
    none, the last j with e_j > 0.  Returns (j, relative margin), the margin
    being the distance from u*S to the nearest edge of token j's interval, / S."""
    c = np.cumsum(e)
    target = u * S
    j = int(np.searchsorted(c, target, side="right"))
    if j >= len(e):
        j = int(np.nonzero(e > 0)[0][-1])
        return j, 0.0
    lo = c[j - 1] if j > 0 else 0.0
    return j, min(target - lo, c[j] - target) / S


def linear_keep_count(n: int, t: int, t_total: int) -> int:
    """k_t = ceil(n * t / T): the linear keep schedule (R-keep)."""
    return min(n, -(-n * t // t_total))


def keep_set(pmax, k):
    """Top-k positions by pmax, ties to the lower index (R-keep).

    Returns (bool mask [N], relative margin between the k-th and (k+1)-th pmax)."""
    pmax = np.asarray(pmax, dtype=np.float64)
    n = len(pmax)
    order = np.lexsort((np.arange(n), -pmax))
    keep = np.zeros(n, dtype=bool)
    keep[order[:k]] = True
    if 0 < k < n:
        a, b = pmax[order[k - 1]], pmax[order[k]]
        margin = (a - b) / max(abs(a), 1e-300)
    else:
        margin = math.inf
    return keep, margin


def keep_entropy_budget(ent, budget):
    """Entropy-ordered locking of [P1 四] (R-budget).

    Positions are taken in order of increasing entropy (ties -> lower index);
    the first (most certain) one is always locked, and each later one while
    the running sum of entropies, this position included, is <= budget.
    Returns (bool mask [N], relative margin: the distance of the running sum
    at the first rejected position from the budget, inf if none is
    rejected)."""
    ent = np.asarray(ent, dtype=np.float64)
    n = len(ent)
    order = np.lexsort((np.arange(n), ent))
    keep = np.zeros(n, dtype=bool)
    run = 0.0
    for pos, i in enumerate(order):
        if pos > 0 and run + ent[i] > budget:
            return keep, ((run + ent[i]) - budget) / max(abs(budget), 1e-300)
        run += ent[i]
        keep[i] = True
    return keep, math.inf


def anneal_temperature(t: int, t_total: int, t_start: float = 0.8, t_end: float = 0.4) -> float:
    """Linear temperature anneal of [P1 四] (R-anneal): t_start at round 1,
    t_end at round t_total."""
    if t_total <= 1:
        return float(t_end)
    return float(t_start + (t_end - t_start) * (t - 1) / (t_total - 1))


def argmax_tokens(logits):
    """The most likely token per position, ties -> lower index: [N, V] -> [N]."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int64)


def stop_two_rounds(mean_h_prev, mean_h, argmax_prev, argmax, tau=0.005):
    """Adaptive stop of [P1 四] (R-stop2): both rounds' mean entropy below tau
    and an unchanged argmax sequence.  The first round has no previous one."""
    if argmax_prev is None or mean_h_prev is None:
        return False
    return bool(mean_h_prev < tau and mean_h < tau and np.array_equal(argmax_prev, argmax))


def sample_canvas(logits, *, seed, step, block, req, temperature, logit_scale,
                  keep_k, stop_threshold, keep_budget=None):
    """Sampler for one canvas: stats, Philox sample, keep, re-noise, stop.

    logits [N, V].  Returns dict with x_hat, pmax, H, keep, x_new, mean_H, stop,
    argmax (of z, ties -> lower index) and the decision margins (sample_margin
    [N], keep_margin, stop_margin, argmax_margin [N]: the gap between the two
    largest z relative to max(|z_max|, 1)).
    stop_threshold < 0 disables the stop test.  keep_budget=None keeps the
    keep_k most confident positions; a number keeps the entropy-budget set
    (R-budget) and ignores keep_k.
    """
    n, vocab = logits.shape
    words = sampler_words(seed, np.arange(n), step, block, req)
    u = unit_uniform(words[:, 0])
    renoise = uniform_token(words[:, 1], vocab)
    x_hat = np.empty(n, dtype=np.int64)
    pmax = np.empty(n)
    ent = np.empty(n)
    smargin = np.empty(n)
    amax = np.empty(n, dtype=np.int64)
    amargin = np.empty(n)
    for i in range(n):
        st = position_stats(logits[i], temperature, logit_scale)
        pmax[i], ent[i] = st["pmax"], st["H"]
        amax[i] = argmax_tokens(st["z"])
        top2 = np.sort(st["z"])[-2:] if vocab > 1 else np.array([-np.inf, st["z"][0]])
        amargin[i] = (top2[1] - top2[0]) / max(abs(top2[1]), 1.0)
        if temperature == 0.0:
            x_hat[i] = int(np.argmax(st["z"]))       # first maximum = lower index
            smargin[i] = math.inf
        else:
            x_hat[i], smargin[i] = inverse_cdf(st["e"], st["S"], u[i])
    if keep_budget is None:
        keep, kmargin = keep_set(pmax, keep_k)
    else:
        keep, kmargin = keep_entropy_budget(ent, keep_budget)
    x_new = np.where(keep, x_hat, renoise)
    mean_h = float(ent.mean())
    stop = bool(stop_threshold >= 0 and mean_h < stop_threshold)
    smg = abs(mean_h - stop_threshold) / max(abs(stop_threshold), 1e-300) if stop_threshold >= 0 else math.inf
    return dict(x_hat=x_hat, pmax=pmax, H=ent, keep=keep, x_new=x_new, renoise=renoise,
                mean_H=mean_h, stop=stop, sample_margin=smargin, keep_margin=kmargin,
                stop_margin=smg, argmax=amax, argmax_margin=amargin)


# ----------------------------------------------------------------------------
# The model and its block-autoregressive driver ([P1 一/二/四], [P2], [P3]).
# ----------------------------------------------------------------------------

@dataclass
class OracleModel:
    """Weights in float64 ([out, in] matrices) and per-request KV caches.

    cfg keys: n_layers, d_model, n_heads, n_kv_heads, head_dim, n_experts,
    top_k, d_ff, vocab, canvas, rope_base, rms_eps.
    weights: embed [V,d], w_sc [d,d], final_norm [d], layers: list of dicts
    attn_norm [d], wq [Hq*hd,d], wk/wv [Hkv*hd,d], wo [d,Hq*hd], ffn_norm [d],
    router_w [E,d], router_b [E] or None, w_gate/w_up [E,F,d], w_down [E,d,F].
    """
    cfg: dict
    weights: dict
    k_cache: dict = field(default_factory=dict)   # req -> list over layers of [Hkv, P, hd]
    v_cache: dict = field(default_factory=dict)

    def length(self, req):
        return 0 if req not in self.k_cache else self.k_cache[req][0].shape[1]

    def _ensure(self, req):
        c = self.cfg
        if req not in self.k_cache:
            z = lambda: np.zeros((c["n_kv_heads"], 0, c["head_dim"]))
            self.k_cache[req] = [z() for _ in range(c["n_layers"])]
            self.v_cache[req] = [z() for _ in range(c["n_layers"])]

    def set_kv(self, req, layer, k, v):
        """Replace request req's cache of one layer by k, v [Hkv, P, hd]."""
        self._ensure(req)
        self.k_cache[req][layer] = np.asarray(k, np.float64)
        self.v_cache[req][layer] = np.asarray(v, np.float64)

    def truncate(self, req, length):
        self._ensure(req)
        for l in range(self.cfg["n_layers"]):
            self.k_cache[req][l] = self.k_cache[req][l][:, :length]
            self.v_cache[req][l] = self.v_cache[req][l][:, :length]

    def layer(self, h, li, req, pos, causal, trace=None):
        """One transformer layer on the n rows of h at positions pos.

        Keys are the request's cache [0, P) followed by the n new rows.  With
        causal=True new row i sees cache + new rows <= i (prompt encoding and
        canvas hand-off, [P1 二], [P2 架构基础]); with causal=False every new row
        sees everything (the bidirectional canvas).  Returns (h_out, k_new, v_new).
        If trace is a dict it receives the MoE input and the router margins
        (recorded only; the arithmetic is unchanged).
        """
        c, L = self.cfg, self.weights["layers"][li]
        hq, hkv, hd = c["n_heads"], c["n_kv_heads"], c["head_dim"]
        n = h.shape[0]
        x = rms_norm(h, L["attn_norm"], c["rms_eps"])
        q = (x @ L["wq"].T).reshape(n, hq, hd).transpose(1, 0, 2)
        k = (x @ L["wk"].T).reshape(n, hkv, hd).transpose(1, 0, 2)
        v = (x @ L["wv"].T).reshape(n, hkv, hd).transpose(1, 0, 2)
        q = rope(q, pos, c["rope_base"])
        k = rope(k, pos, c["rope_base"])
        kc, vc = self.k_cache[req][li], self.v_cache[req][li]
        p_len = kc.shape[1]
        kk = np.concatenate([kc, k], axis=1)
        vv = np.concatenate([vc, v], axis=1)
        allowed = None
        if causal:
            allowed = np.arange(p_len + n)[None, :] <= (p_len + np.arange(n))[:, None]
        o = attention(q, kk, vv, allowed).transpose(1, 0, 2).reshape(n, hq * hd)
        h = h + o @ L["wo"].T
        x = rms_norm(h, L["ffn_norm"], c["rms_eps"])
        if trace is not None:
            ids, _, g, margin = router(x, L["router_w"], L.get("router_b"), c["top_k"])
            trace.update(moe_in=x, router_ids=ids, router_logits=g, router_margin=margin, h_attn=h)
        h = h + moe(x, L, c["top_k"])
        return h, k, v

    def embed_tokens(self, tokens, prev_pred=None):
        """Token embedding plus the self-conditioning term (R-sc, [P1 二])."""
        E = self.weights["embed"]
        h = E[np.asarray(tokens)].astype(np.float64)
        if prev_pred is not None:
            h = h + E[np.asarray(prev_pred)].astype(np.float64) @ np.asarray(self.weights["w_sc"], np.float64).T
        return h

    def encode_causal(self, req, tokens):
        """Causal encode of tokens at positions P..P+n-1, appending their K/V
        (prompt prefill, and the block hand-off R-append)."""
        self._ensure(req)
        p0 = self.length(req)
        tokens = np.asarray(tokens)
        pos = p0 + np.arange(len(tokens))
        h = self.embed_tokens(tokens)
        new_k, new_v = [], []
        for li in range(self.cfg["n_layers"]):
            h, k, v = self.layer(h, li, req, pos, causal=True)
            new_k.append(k)
            new_v.append(v)
        for li in range(self.cfg["n_layers"]):
            self.k_cache[req][li] = np.concatenate([self.k_cache[req][li], new_k[li]], axis=1)
            self.v_cache[req][li] = np.concatenate([self.v_cache[req][li], new_v[li]], axis=1)
        return h

    def denoise_forward(self, req, canvas, prev_pred=None, n_layers=None, return_hidden=False):
        """One forward pass over a canvas: embed + self-cond, all layers
        (bidirectional in the canvas, over the whole cache), final norm, tied
        LM head.  Returns logits [N, V] (and the residual stream if asked)."""
        self._ensure(req)
        c = self.cfg
        canvas = np.asarray(canvas)
        pos = self.length(req) + np.arange(len(canvas))
        h = self.embed_tokens(canvas, prev_pred)
        nl = c["n_layers"] if n_layers is None else n_layers
        for li in range(nl):
            h, _, _ = self.layer(h, li, req, pos, causal=False)
        x = rms_norm(h, self.weights["final_norm"], c["rms_eps"])
        logits = lm_head(x, self.weights["embed"])
        return (logits, h) if return_hidden else logits

    def ar_next_logits(self, req, token):
        """AR mode (R-ar): append one token to the request's cache by a causal
        pass and return the logits [V] of the token that follows it."""
        h = self.encode_causal(req, [int(token)])
        x = rms_norm(h, self.weights["final_norm"], self.cfg["rms_eps"])
        return lm_head(x, self.weights["embed"])[0]

    def denoise_step(self, req, canvas, prev_pred, *, step, block, seed, temperature,
                     logit_scale, keep_k, stop_threshold, keep_budget=None):
        logits = self.denoise_forward(req, canvas, prev_pred)
        out = sample_canvas(logits, seed=seed, step=step, block=block, req=req,
                            temperature=temperature, logit_scale=logit_scale,
                            keep_k=keep_k, stop_threshold=stop_threshold,
                            keep_budget=keep_budget)
        out["logits"] = logits
        return out

    def generate_block(self, req, *, seed, block, max_steps, schedule_steps,
                       temperature, logit_scale_growth=1.0, stop_threshold=-1.0,
                       append=True, keep_budget=None, temperature_end=None,
                       two_round_stop=False):
        """One block ([P1 一/四], [P2 运作机制], [P3]): random canvas, up to
        max_steps denoise steps with the linear keep schedule over
        schedule_steps, stop on mean entropy, output the last x_hat, then the
        causal hand-off of the block into the cache.  Returns (tokens, steps, trace).
        keep_budget: the entropy-budget keep (R-budget) instead of the schedule.
        temperature_end: the linear anneal (R-anneal) from `temperature` at
        step 1 to it at step max_steps; each step's temperature is recorded in
        its trace entry.
        two_round_stop: the stop of R-stop2 with tau = stop_threshold (< 0
        disables it) in place of the one-round mean-entropy test."""
        n, vocab = self.cfg["canvas"], self.cfg["vocab"]
        canvas = init_canvas(seed, n, vocab, block, req)
        prev = None
        trace = []
        out_tokens, steps = None, 0
        for t in range(1, max_steps + 1):
            temp = temperature if temperature_end is None else \
                anneal_temperature(t, max_steps, temperature, temperature_end)
            r = self.denoise_step(req, canvas, prev, step=t, block=block, seed=seed,
                                  temperature=temp,
                                  logit_scale=logit_scale_growth ** (t - 1),
                                  keep_k=linear_keep_count(n, t, schedule_steps),
                                  stop_threshold=stop_threshold, keep_budget=keep_budget)
            r["canvas_in"] = canvas.copy()
            r["temperature"] = temp
            if two_round_stop:
                prev_r = trace[-1] if trace else None
                r["stop"] = stop_threshold >= 0 and prev_r is not None and stop_two_rounds(
                    prev_r["mean_H"], r["mean_H"], prev_r["argmax"], r["argmax"], tau=stop_threshold)
                r["stop_margin"] = math.inf if prev_r is None or stop_threshold < 0 else \
                    min(abs(prev_r["mean_H"] - stop_threshold), abs(r["mean_H"] - stop_threshold)) / \
                    max(stop_threshold, 1e-300)
            trace.append(r)
            steps = t
            if r["stop"] or t == max_steps:
                out_tokens = r["x_hat"].copy()
                break
            prev = r["x_hat"]
            canvas = r["x_new"]
        if append:
            self.encode_causal(req, out_tokens)
        return out_tokens, steps, trace


def lm_head(x, embed, chunk=16384):
    """Tied LM head: logits = x E^T ([P1 五]: softmax over the 262k vocabulary
    follows it).  Evaluated in vocabulary chunks only to bound the float64
    temporaries; each logit is one plain dot product."""
    x = np.asarray(x, np.float64)
    out = np.empty((x.shape[0], embed.shape[0]))
    for v0 in range(0, embed.shape[0], chunk):
        out[:, v0:v0 + chunk] = x @ np.asarray(embed[v0:v0 + chunk], np.float64).T
    return out


def max_abs_rel(a, b):
    """max|a - b| / max|b| over a tensor (the comparison metric of the tests)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))
