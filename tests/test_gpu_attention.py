"""Attention at full width (d 2816, 16 query / 8 KV heads of 256) against the
oracle, isolated from routing: the experts' down projections are zero, so the
MoE adds exactly 0 on both sides and the layer output is
embedding + O-proj(attention(RoPE(QKV))).  Covers the canvas step over a long
cache (split-KV path, up to the 8192-position prompt of the full-depth
workload), the causal encode of ragged prompts, and two requests of
different lengths in one batch.  With 16 query heads over 8 KV heads the
pair kernel runs (two query heads per CTA pair, 128-key tiles); with as many
KV heads as query heads, the one-CTA-per-head kernel (64-key tiles).
Tolerance: max-abs-rel 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import max_abs_rel, to_np

FULL = dict(synth.FULL_SHAPE, n_layers=1, vocab=4096)
TOL = 2e-2


MHA = dict(FULL, n_heads=8, n_kv_heads=8)


def _model(max_batch, max_ctx, seed=21, model=FULL):
    w = synth.make_weights(model, seed=seed, dtype="bf16", router_bias=True, device="cuda")
    w["layers"][0]["w_down"].zero_()
    om = O.OracleModel(dict(model), synth.to_numpy_weights(w))
    return w, om


def _step_hidden(dg, h, req, canvas):
    n, d = FULL["canvas"], FULL["d_model"]
    hid = torch.zeros((len(req) * n, d), device="cuda")
    dg.dg_denoise_step(h, req, canvas.cuda(), None, 1, dg.sampler_params(keep_k=1), dg.step_out(), hidden_out=hid)
    dg.dg_synchronize(h)
    return to_np(hid)


@pytest.mark.gpu
@pytest.mark.parametrize("cache_len", [64, 2048, 8192])
def test_canvas_attention_over_long_cache(dg, cache_len):
    w, om = _model(1, cache_len + 256)
    h = dg.dg_create(FULL, w, dtype="bf16", max_batch=1, max_ctx=cache_len + 256)
    k, v = synth.normal_kv(FULL["n_kv_heads"], cache_len, FULL["head_dim"], seed=cache_len, dtype="bf16",
                           device="cuda")
    dg.dg_set_kv(h, 0, 0, k, v)
    dg.dg_set_length(h, 0, cache_len)
    om.set_kv(0, 0, k.float().cpu().numpy(), v.float().cpu().numpy())
    canvas = synth.uniform_tokens(FULL["canvas"], FULL["vocab"], seed=3)
    got = _step_hidden(dg, h, [0], canvas[None])
    ref, _, _ = om.layer(om.embed_tokens(canvas.numpy()), 0, 0, cache_len + np.arange(FULL["canvas"]), causal=False)
    err = max_abs_rel(got, ref)
    assert err < TOL, err
    h.close()


@pytest.mark.gpu
def test_canvas_attention_one_cta_per_head(dg):
    cache_len = 2048
    w, om = _model(1, cache_len + 256, model=MHA)
    h = dg.dg_create(MHA, w, dtype="bf16", max_batch=1, max_ctx=cache_len + 256)
    k, v = synth.normal_kv(MHA["n_kv_heads"], cache_len, MHA["head_dim"], seed=7, dtype="bf16", device="cuda")
    dg.dg_set_kv(h, 0, 0, k, v)
    dg.dg_set_length(h, 0, cache_len)
    om.set_kv(0, 0, k.float().cpu().numpy(), v.float().cpu().numpy())
    canvas = synth.uniform_tokens(MHA["canvas"], MHA["vocab"], seed=8)
    got = _step_hidden(dg, h, [0], canvas[None])
    ref, _, _ = om.layer(om.embed_tokens(canvas.numpy()), 0, 0, cache_len + np.arange(MHA["canvas"]), causal=False)
    err = max_abs_rel(got, ref)
    assert err < TOL, err
    h.close()


@pytest.mark.gpu
@pytest.mark.parametrize("model", [FULL, MHA], ids=["gqa_pairs", "one_cta_per_head"])
def test_causal_prefill_ragged_then_canvas_batch_of_two(dg, model):
    w, om = _model(2, 1024, model=model)
    h = dg.dg_create(model, w, dtype="bf16", max_batch=2, max_ctx=1024, max_tokens=512)
    p0 = synth.uniform_tokens(300, model["vocab"], seed=4)      # ragged: not a multiple of 64 or 128
    p1 = synth.uniform_tokens(517, model["vocab"], seed=5)      # chunked: 517 > max_tokens / batch
    dg.dg_prefill_prompt(h, [1], p0[None].cuda())
    dg.dg_prefill_prompt(h, [0], p1[None].cuda())
    om.encode_causal(1, p0.numpy())
    om.encode_causal(0, p1.numpy())
    assert dg.dg_get_length(h, 1) == 300 and dg.dg_get_length(h, 0) == 517
    canvas = synth.uniform_tokens(model["canvas"], model["vocab"], seed=6, batch=2)
    got = _step_hidden(dg, h, [1, 0], canvas)
    n = model["canvas"]
    for b, req in enumerate([1, 0]):
        plen = om.length(req)
        ref, _, _ = om.layer(om.embed_tokens(canvas[b].numpy()), 0, req, plen + np.arange(n), causal=False)
        err = max_abs_rel(got[b * n:(b + 1) * n], ref)
        assert err < TOL, (req, err)
    h.close()
