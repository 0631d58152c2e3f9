"""The fused LM head -> sampler ([P1 五]: the 262k-vocabulary softmax is a large
share of the per-step cost).  Without a logits buffer from the caller, a step
never writes the fp32 logits: the LM head's epilogue reduces each token's
logits over 32-entry vocabulary groups to (max, first arg-max, sum exp, sum
exp * z), and the sampler merges those records and recomputes only the 32
logits of the group that holds its Philox draw.

Checked on one full-width layer (vocabulary 262144, 8192 groups) at T 1.0, 0.8
and 0 (arg-max), against the same step with the logits materialised (same
GEMM, so the same fp32 logits) and against the oracle's sampler on those
logits: pmax and entropy within 1e-5, the arg-max exactly, x_hat, the keep set
and the re-noised canvas by the margin rule.
"""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import check_decisions, to_np

W = synth.WORKLOADS["layer_bf16"]
M = W["model"]


def _outs(n):
    dev = "cuda"
    return dict(x_hat=torch.full((1, n), -1, dtype=torch.int32, device=dev), pmax=torch.zeros((1, n), device=dev),
                entropy=torch.zeros((1, n), device=dev), keep=torch.zeros((1, n), dtype=torch.int32, device=dev),
                mean_entropy=torch.zeros(1, device=dev), stop=torch.zeros(1, dtype=torch.int32, device=dev),
                argmax=torch.full((1, n), -1, dtype=torch.int32, device=dev))


@pytest.mark.gpu
@pytest.mark.parametrize("temperature,scale", [(1.0, 1.0), (0.8, 2.25), (0.0, 1.0)])
def test_fused_head_matches_materialised_logits_and_oracle(dg, temperature, scale):
    w = synth.make_weights(M, seed=W["seed"], dtype="bf16", router_bias=True, device="cuda")
    k, v = synth.normal_kv(M["n_kv_heads"], W["cache_len"], M["head_dim"], seed=W["seed"] + 50, dtype="bf16",
                           device="cuda")
    h = dg.dg_create(M, w, dtype="bf16", max_batch=1, max_ctx=W["cache_len"] + M["canvas"])
    dg.dg_set_kv(h, 0, 0, k, v)
    dg.dg_set_length(h, 0, W["cache_len"])
    n, V = M["canvas"], M["vocab"]
    canvas0 = synth.uniform_tokens(n, V, seed=W["seed"] + 11)[None].cuda()
    seed, step, keep_k = 9, 3, 96
    sp = dg.sampler_params(temperature=temperature, logit_scale=scale, keep_k=keep_k, stop_threshold=0.5, seed=seed,
                           block=2)
    logits = torch.empty((1, n, V), device="cuda")
    A, Bo = _outs(n), _outs(n)
    ca, cb = canvas0.clone(), canvas0.clone()
    dg.dg_denoise_step(h, [0], ca, None, step, sp, dg.step_out(**A), logits_out=logits)
    dg.dg_denoise_step(h, [0], cb, None, step, sp, dg.step_out(**Bo))      # fused: no logits buffer
    dg.dg_synchronize(h)
    a = {kk: to_np(t)[0] for kk, t in A.items()}
    b = {kk: to_np(t)[0] for kk, t in Bo.items()}
    lg = to_np(logits)[0].astype(np.float64)
    h.close()
    # statistics: the same logits, merged in another order
    assert np.allclose(b["pmax"], a["pmax"], rtol=1e-5, atol=1e-9)
    assert np.allclose(b["entropy"], a["entropy"], rtol=1e-5, atol=1e-6)
    assert np.array_equal(b["argmax"], a["argmax"])
    # the oracle's sampler on the materialised logits decides the samples
    ref = O.sample_canvas(lg, seed=seed, step=step, block=2, req=0, temperature=temperature, logit_scale=scale,
                          keep_k=keep_k, stop_threshold=0.5)
    assert np.allclose(b["pmax"], ref["pmax"], rtol=1e-4, atol=1e-9)
    assert np.allclose(b["entropy"], ref["H"], rtol=1e-4, atol=1e-5)
    low = check_decisions(b["x_hat"], ref["x_hat"], ref["sample_margin"], "fused x_hat")
    assert low <= 1
    check_decisions(b["argmax"], ref["argmax"], ref["argmax_margin"], "fused argmax")
    if ref["keep_margin"] > 1e-5:
        assert np.array_equal(b["keep"].astype(bool), ref["keep"])
    keep = b["keep"].astype(bool)
    assert keep.sum() == keep_k
    got_canvas = to_np(cb)[0]
    assert np.array_equal(got_canvas[keep], b["x_hat"][keep])
    assert np.array_equal(got_canvas[~keep], ref["renoise"][~keep])
    assert abs(float(b["mean_entropy"]) - float(np.mean(b["entropy"].astype(np.float64)))) < 1e-5
