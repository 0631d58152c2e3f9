"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module holds workload shapes and random-input recipes only: it does none of
the method's arithmetic.  Every tensor is drawn from a seeded torch generator,
so the CUDA path and the CPU oracle are handed bit-identical inputs.

Workloads (named by what they are):
  tiny_fp32   2 layers, d 256, 4/2 heads of 64, 8 experts top-2, FFN 512,
              vocab 1024, canvas 32, prompt 32; fp32 weights.
  layer_bf16  1 full-width layer: d 2816, 16/8 heads of 256, 128 experts
              top-8, FFN 704, vocab 262144, canvas 256; bf16 weights; router
              bias N(0,1); a 2048-position N(0,1) KV cache.
  sampler     logits [B, 256, 262144] fp32 = Gumbel(0,1) + h * onehot(r),
              h ~ U(0,12), r ~ U[0,V); B in {1, 16, 64}; T 0.8; k in
              {64, 128, 192}; stop threshold 0.1.
  full_b1     30 layers of the full-width shape, prompt 8192, one canvas,
              up to 48 steps, linear keep over 48, stop 0.1 nats, logit
              scale 1.5^(t-1).
  full_b16    the same model; 16 requests with 4096-token prompts, 4 blocks
              of 12 fixed steps each (stop disabled).
"""
from __future__ import annotations

import torch

FULL_SHAPE = dict(d_model=2816, n_heads=16, n_kv_heads=8, head_dim=256, n_experts=128,
                  top_k=8, d_ff=704, vocab=262144, canvas=256, rope_base=10000.0,
                  rms_eps=1e-6)

WORKLOADS = {
    "tiny_fp32": dict(model=dict(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64,
                                 n_experts=8, top_k=2, d_ff=512, vocab=1024, canvas=32,
                                 rope_base=10000.0, rms_eps=1e-6),
                      dtype="fp32", router_bias=False, prompt_len=32, batch=1,
                      sampler=dict(temperature=1.0, max_steps=4, schedule_steps=4,
                                   stop_threshold=0.05, logit_scale_growth=1.0, seed=0),
                      seed=0),
    "layer_bf16": dict(model=dict(n_layers=1, **FULL_SHAPE), dtype="bf16", router_bias=True,
                       cache_len=2048, batch=1,
                       sampler=dict(temperature=1.0, max_steps=1, schedule_steps=1,
                                    stop_threshold=0.1, logit_scale_growth=1.0, seed=1),
                       seed=1),
    "sampler": dict(vocab=262144, canvas=256, batches=(1, 16, 64), temperature=0.8,
                    keep=(64, 128, 192), stop_threshold=0.1, peak_max=12.0, seed=2),
    "full_b1": dict(model=dict(n_layers=30, **FULL_SHAPE), dtype="bf16", router_bias=True,
                    prompt_len=8192, batch=1,
                    sampler=dict(temperature=1.0, max_steps=48, schedule_steps=48,
                                 stop_threshold=0.1, logit_scale_growth=1.5, seed=3),
                    seed=3),
    "full_b16": dict(model=dict(n_layers=30, **FULL_SHAPE), dtype="bf16", router_bias=True,
                     prompt_len=4096, batch=16, blocks=4,
                     sampler=dict(temperature=1.0, max_steps=12, schedule_steps=12,
                                  stop_threshold=-1.0, logit_scale_growth=1.0, seed=4),
                     seed=4),
}

WEIGHT_STD = 0.02


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, g, device, dtype):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(dtype)


def make_weights(model: dict, *, seed: int, dtype: str, router_bias: bool,
                 device="cpu", layers=None):
    """Random-init weights of the given shape, in the library's layouts:
    every matrix is [out, in] row-major; norms (ones) and router bias are fp32.

    layers: optional iterable of layer indices to materialise (others None),
    so that a host-side check can draw one layer of a deep model.  Each layer
    draws from its own generator (seed, layer), so any subset is identical to
    the same layers of the full draw.
    """
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    d, hq, hkv, hd = model["d_model"], model["n_heads"], model["n_kv_heads"], model["head_dim"]
    e, f, v = model["n_experts"], model["d_ff"], model["vocab"]
    g = _gen(seed * 1000 + 999, device)
    w = dict(embed=_normal((v, d), WEIGHT_STD, g, device, tdt),
             w_sc=_normal((d, d), WEIGHT_STD, g, device, tdt),
             final_norm=torch.ones(d, device=device, dtype=torch.float32))
    want = set(range(model["n_layers"])) if layers is None else set(layers)
    w["layers"] = []
    for li in range(model["n_layers"]):
        if li not in want:
            w["layers"].append(None)
            continue
        gl = _gen(seed * 1000 + li, device)
        w["layers"].append(dict(
            attn_norm=torch.ones(d, device=device, dtype=torch.float32),
            wq=_normal((hq * hd, d), WEIGHT_STD, gl, device, tdt),
            wk=_normal((hkv * hd, d), WEIGHT_STD, gl, device, tdt),
            wv=_normal((hkv * hd, d), WEIGHT_STD, gl, device, tdt),
            wo=_normal((d, hq * hd), WEIGHT_STD, gl, device, tdt),
            ffn_norm=torch.ones(d, device=device, dtype=torch.float32),
            router_w=_normal((e, d), WEIGHT_STD, gl, device, tdt),
            router_b=(_normal((e,), 1.0, gl, device, torch.float32) if router_bias else None),
            w_gate=_normal((e, f, d), WEIGHT_STD, gl, device, tdt),
            w_up=_normal((e, f, d), WEIGHT_STD, gl, device, tdt),
            w_down=_normal((e, d, f), WEIGHT_STD, gl, device, tdt),
        ))
    return w


def uniform_tokens(n, vocab, *, seed, device="cpu", batch=None):
    """Prompt / canvas tokens uniform over [0, vocab), int32."""
    g = _gen(seed, device)
    shape = (n,) if batch is None else (batch, n)
    return torch.randint(0, vocab, shape, generator=g, device=device, dtype=torch.int32)


def normal_kv(n_kv_heads, length, head_dim, *, seed, dtype, device="cpu"):
    """An N(0,1) K/V cache [Hkv, length, hd] (the layer_bf16 prompt cache)."""
    g = _gen(seed, device)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    k = torch.randn((n_kv_heads, length, head_dim), generator=g, device=device).to(tdt)
    v = torch.randn((n_kv_heads, length, head_dim), generator=g, device=device).to(tdt)
    return k, v


def peaked_logits(batch, n, vocab, *, seed, peak_max=12.0, device="cpu"):
    """Sampler workload logits [batch, n, vocab] fp32: Gumbel(0,1) noise plus a
    peak of height h ~ U(0, peak_max) at a uniform-random token per position.
    Returns (logits, peak_token [batch, n], peak_height [batch, n])."""
    g = _gen(seed, device)
    u = torch.rand((batch, n, vocab), generator=g, device=device, dtype=torch.float32)
    u.clamp_(min=1e-30)
    logits = -torch.log(-torch.log(u))
    r = torch.randint(0, vocab, (batch, n), generator=g, device=device)
    h = torch.rand((batch, n), generator=g, device=device) * peak_max
    logits.scatter_add_(2, r[..., None], h[..., None])
    return logits, r.to(torch.int32), h


def to_numpy_weights(w):
    """Torch weights -> numpy float32 arrays (bf16 values are exact in fp32)."""
    def cv(t):
        return None if t is None else t.detach().to("cpu", torch.float32).numpy()
    out = {k: cv(w[k]) for k in ("embed", "w_sc", "final_norm")}
    out["layers"] = [None if L is None else {k: cv(t) for k, t in L.items()} for L in w["layers"]]
    return out
