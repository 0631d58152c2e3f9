"""AR-mode decode ([P1 七]: the diffusion model's weights run unchanged as an
autoregressive model) through dg_ar_step, against the oracle's AR step.

Each call encodes one token per request causally at the end of its cache and
returns the logits of the next token (final norm + tied LM head).  Checked: the
logits (1e-4 for fp32, 2e-2 for bf16, max-abs-rel), the greedy next token
(bit-exact on the GPU's own logits, and against the oracle's where its top-two
gap is not a rounding tie), the K/V the step appended, and the cache length.
The bf16 cases run the single-token attention kernel: query heads sharing a KV
head (2 and 4 per KV head), two requests of different lengths in one batch,
and the full-width layer over a 2048-position cache.
"""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import max_abs_rel, to_np


def _gpu_weights(w):
    wd = {k: v.cuda() for k, v in w.items() if k != "layers"}
    wd["layers"] = [{k: (None if v is None else v.cuda()) for k, v in L.items()} for L in w["layers"]]
    return wd


def _run(dg, model, dtype, prompts, steps, tol, seed, max_ctx=1024, cache=None):
    """prompts: token lists per request (or None with `cache` = (k, v, length) for request 0)."""
    w = synth.make_weights(model, seed=seed, dtype=dtype, router_bias=True)
    om = O.OracleModel(dict(model), synth.to_numpy_weights(w))
    wd = _gpu_weights(w)
    B = len(prompts)
    h = dg.dg_create(model, wd, dtype=dtype, max_batch=B, max_ctx=max_ctx)
    req = list(range(B))
    if cache is not None:
        k, v, n = cache
        dg.dg_set_kv(h, 0, 0, k.cuda(), v.cuda())
        dg.dg_set_length(h, 0, n)
        om.set_kv(0, 0, k.float().numpy(), v.float().numpy())
    else:
        for r, p in enumerate(prompts):
            dg.dg_prefill_prompt(h, [r], torch.tensor([p], dtype=torch.int32).cuda())
            om.encode_causal(r, np.array(p))
    V = model["vocab"]
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, V, size=B).astype(np.int32)
    for s in range(steps):
        logits = torch.zeros((B, V), device="cuda")
        nxt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        before = [dg.dg_get_length(h, r) for r in req]
        dg.dg_ar_step(h, req, torch.from_numpy(tok).cuda(), logits, nxt)
        dg.dg_synchronize(h)
        got = to_np(logits).astype(np.float64)
        for r in req:
            assert dg.dg_get_length(h, r) == before[r] + 1
            ref = om.ar_next_logits(r, int(tok[r]))
            err = max_abs_rel(got[r], ref)
            assert err < tol, f"step {s} req {r}: logits max-abs-rel {err}"
            # greedy token: exactly the argmax of the GPU's own logits (first of equals) ...
            assert int(to_np(nxt)[r]) == int(np.argmax(to_np(logits)[r]))
            # ... and the oracle's argmax unless its top-two gap is within the rounding error
            top2 = np.sort(ref)[-2:]
            if top2[1] - top2[0] > 4 * tol * np.max(np.abs(ref)):
                assert int(to_np(nxt)[r]) == int(np.argmax(ref))
        # the K/V the first layer appended at the new position (RoPE'd at P - 1), against the
        # oracle's cache; the input of layer 0 is the embedding, so only this layer's rounding enters
        for r in req:
            P = dg.dg_get_length(h, r)
            kd = torch.empty((model["n_kv_heads"], P, model["head_dim"]),
                             dtype=torch.float32 if dtype == "fp32" else torch.bfloat16, device="cuda")
            vd = torch.empty_like(kd)
            dg.dg_get_kv(h, r, 0, kd, vd)
            dg.dg_synchronize(h)
            kref = om.k_cache[r][0][:, P - 1]
            vref = om.v_cache[r][0][:, P - 1]
            assert max_abs_rel(to_np(kd.float())[:, P - 1], kref) < tol
            assert max_abs_rel(to_np(vd.float())[:, P - 1], vref) < tol
        tok = to_np(nxt).astype(np.int32)
    launches = dg.dg_launch_count(h)
    h.close()
    return launches


@pytest.mark.gpu
def test_ar_step_tiny_fp32(dg):
    W = synth.WORKLOADS["tiny_fp32"]
    M = W["model"]
    prompts = [synth.uniform_tokens(32, M["vocab"], seed=40).tolist(),
               synth.uniform_tokens(45, M["vocab"], seed=41).tolist()]
    _run(dg, M, "fp32", prompts, steps=3, tol=1e-4, seed=42, max_ctx=128)


@pytest.mark.gpu
@pytest.mark.parametrize("hq,hkv", [(2, 1), (4, 1), (8, 4)])
def test_ar_step_bf16_single_token_attention(dg, hq, hkv):
    M = dict(n_layers=2, d_model=256, n_heads=hq, n_kv_heads=hkv, head_dim=256, n_experts=16, top_k=4,
             d_ff=128, vocab=4096, canvas=32, rope_base=10000.0, rms_eps=1e-6)
    prompts = [synth.uniform_tokens(300, M["vocab"], seed=50).tolist(),
               synth.uniform_tokens(517, M["vocab"], seed=51).tolist()]
    _run(dg, M, "bf16", prompts, steps=3, tol=2e-2, seed=52, max_ctx=1024)


@pytest.mark.gpu
def test_ar_step_full_width_layer_over_2048_cache(dg):
    W = synth.WORKLOADS["layer_bf16"]
    M = dict(W["model"])
    k, v = synth.normal_kv(M["n_kv_heads"], W["cache_len"], M["head_dim"], seed=W["seed"] + 60, dtype="bf16")
    _run(dg, M, "bf16", [None], steps=2, tol=2e-2, seed=61, max_ctx=W["cache_len"] + 256,
         cache=(k, v, W["cache_len"]))


@pytest.mark.gpu
def test_ar_step_refuses_full_cache(dg):
    W = synth.WORKLOADS["tiny_fp32"]
    M = W["model"]
    w = _gpu_weights(synth.make_weights(M, seed=1, dtype="fp32", router_bias=False))
    h = dg.dg_create(M, w, dtype="fp32", max_batch=1, max_ctx=64)
    dg.dg_set_length(h, 0, 64)
    logits = torch.zeros((1, M["vocab"]), device="cuda")
    with pytest.raises(dg.DgError) as e:
        dg.dg_ar_step(h, [0], torch.zeros(1, dtype=torch.int32, device="cuda"), logits)
    assert e.value.code == dg.DG_ECAPACITY
    assert dg.dg_get_length(h, 0) == 64
    h.close()
