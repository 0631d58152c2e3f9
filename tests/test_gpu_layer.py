"""Full-width bf16 layer (d 2816, 16/8 heads of 256, 128 experts top-8, FFN
704, vocab 262144, router bias N(0,1), a 2048-position N(0,1) bf16 KV cache,
canvas 256): one denoise step through the C ABI, checked layer-output-wise and
on sampled logits against the float64 oracle (max-abs-rel 2e-2 for bf16).
Plus the tensor-core GEMM alone against a float64 matmul of the same operands."""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import max_abs_rel, to_np

W = synth.WORKLOADS["layer_bf16"]
M = W["model"]
TOL_BF16 = 2e-2
# Router logits carry ~2^-8 relative error from the bf16 MoE input (~0.005 in
# logit units here); decisions closer than 4x that are rounding-order ties.
ROUTER_MARGIN = 0.02


@pytest.mark.gpu
@pytest.mark.parametrize("T,Mr,K", [(1, 128, 64), (31, 200, 128), (256, 384, 2816), (300, 4096, 2816),
                                    (4096, 512, 704), (96, 262144 // 64, 2816)])
def test_tc_gemm_matches_float64_matmul(dg, T, Mr, K):
    g = torch.Generator(device="cuda").manual_seed(T * 7 + Mr)
    x = torch.randn((T, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((Mr, K), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    out = torch.full((T, Mr), float("nan"), device="cuda")
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="bf16", max_batch=1, max_ctx=64)
    dg.dg_selftest_gemm(h, x, w, out)
    dg.dg_synchronize(h)
    ref = x.double().cpu() @ w.double().cpu().T
    err = max_abs_rel(to_np(out), ref.numpy())
    assert err < 1e-3, err
    h.close()


@pytest.mark.gpu
@pytest.mark.parametrize("T,Mr,K", [(256, 8192, 2816), (256, 2816, 4096), (256, 2816, 2816), (37, 384, 192),
                                    (130, 200, 2816), (1, 128, 64)])
def test_split_k_gemm_slices_sum_to_float64_matmul(dg, T, Mr, K):
    """The split-K form of the QKV / O / self-conditioning projections: its
    slices, added in order, equal the product (several tiles, ragged M and T)."""
    g = torch.Generator(device="cuda").manual_seed(T * 5 + Mr)
    x = torch.randn((T, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((Mr, K), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    part = torch.full((8, T, Mr), float("nan"), device="cuda")
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="bf16", max_batch=1, max_ctx=64)
    ns = dg.dg_selftest_gemm_split(h, x, w, part)
    dg.dg_synchronize(h)
    assert 1 <= ns <= 8
    if (T, Mr, K) == (256, 2816, 4096):
        assert ns > 1      # the O-projection shape splits K
    assert not torch.isnan(part[:ns]).any()
    got = part[:ns].double().sum(0)
    ref = x.double().cpu() @ w.double().cpu().T
    err = max_abs_rel(to_np(got), ref.numpy())
    assert err < 1e-3, err
    h.close()


def _layer_setup(dg, hot_experts=0):
    w = synth.make_weights(M, seed=W["seed"], dtype="bf16", router_bias=True, device="cuda")
    if hot_experts:
        # a large bias on a few experts routes every token to them: expert work
        # items of 256 rows next to items of a few rows
        w["layers"][0]["router_b"][:hot_experts] += 8.0
    k, v = synth.normal_kv(M["n_kv_heads"], W["cache_len"], M["head_dim"], seed=W["seed"] + 50, dtype="bf16",
                           device="cuda")
    h = dg.dg_create(M, w, dtype="bf16", max_batch=1, max_ctx=W["cache_len"] + M["canvas"])
    dg.dg_set_kv(h, 0, 0, k, v)
    dg.dg_set_length(h, 0, W["cache_len"])
    om = O.OracleModel(dict(M), synth.to_numpy_weights(w))
    om.set_kv(0, 0, k.float().cpu().numpy(), v.float().cpu().numpy())
    return w, h, om


@pytest.mark.gpu
@pytest.mark.parametrize("hot_experts", [0, 4])
def test_full_width_layer_step(dg, hot_experts):
    w, h, om = _layer_setup(dg, hot_experts)
    n, vocab, d = M["canvas"], M["vocab"], M["d_model"]
    canvas = synth.uniform_tokens(n, vocab, seed=W["seed"] + 1)
    prev = synth.uniform_tokens(n, vocab, seed=W["seed"] + 2)
    rows = np.arange(0, n, 16)
    for use_prev in (False, True):
        logits = torch.zeros((1, n, vocab), device="cuda")
        hid = torch.zeros((n, d), device="cuda")
        touched = torch.zeros(1, dtype=torch.int32, device="cuda")
        sp = dg.sampler_params(temperature=1.0, keep_k=64, stop_threshold=0.1, seed=1)
        dg.dg_denoise_step(h, [0], canvas[None].cuda(), prev[None].cuda() if use_prev else None, 1, sp,
                           dg.step_out(experts_touched=touched), logits_out=logits, hidden_out=hid)
        dg.dg_synchronize(h)
        pos = W["cache_len"] + np.arange(n)
        hx = om.embed_tokens(canvas.numpy(), prev.numpy() if use_prev else None)
        tr = {}
        ref_h, _, _ = om.layer(hx, 0, 0, pos, causal=False, trace=tr)
        # Tokens whose 8th/9th router logits are closer than the bf16 error of
        # the router input may legitimately pick another expert: compare the
        # rest, and require them to be the large majority.
        safe = tr["router_margin"] > ROUTER_MARGIN
        assert safe.mean() > 0.6, f"only {safe.mean():.2f} of tokens have a router margin > {ROUTER_MARGIN}"
        got_h = to_np(hid)
        den = np.max(np.abs(ref_h))
        err_h = float(np.max(np.abs(got_h[safe] - ref_h[safe])) / den)
        assert err_h < TOL_BF16, f"layer output max-abs-rel {err_h} (self-cond={use_prev})"
        r = rows[safe[rows]]
        x = O.rms_norm(ref_h[r], om.weights["final_norm"], M["rms_eps"])
        ref_l = O.lm_head(x, om.weights["embed"])
        err_l = max_abs_rel(to_np(logits)[0][r], ref_l)
        assert err_l < TOL_BF16, f"logits max-abs-rel {err_l}"
        assert 1 <= int(touched.item()) <= M["n_experts"]
        if hot_experts:
            assert (tr["router_ids"] < hot_experts).sum(1).min() == hot_experts
    h.close()
