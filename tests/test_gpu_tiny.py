"""Tiny fp32 denoiser end to end (2 layers, d 256, 4/2 heads of 64, 8 experts
top-2, FFN 512, vocab 1024, canvas 32, prompt 32, 4 steps, T 1.0, linear keep,
stop 0.05, Philox seed 0): prefill, each denoise step, the block loop and the
hand-off into the KV cache, all through the C ABI, against the oracle.
Logits must agree to max-abs-rel 1e-4; integer decisions exactly (margin rule)."""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import check_decisions, max_abs_rel, to_np

W = synth.WORKLOADS["tiny_fp32"]
M = W["model"]
S = W["sampler"]


def _setup(dg):
    w = synth.make_weights(M, seed=W["seed"], dtype="fp32", router_bias=W["router_bias"])
    prompt = synth.uniform_tokens(W["prompt_len"], M["vocab"], seed=W["seed"] + 100)
    om = O.OracleModel(dict(M), synth.to_numpy_weights(w))
    om.encode_causal(0, prompt.numpy())
    wd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in w.items() if k != "layers"}
    wd["layers"] = [{k: (None if v is None else v.cuda()) for k, v in L.items()} for L in w["layers"]]
    h = dg.dg_create(M, wd, dtype="fp32", max_batch=2, max_ctx=128)
    dg.dg_prefill_prompt(h, [0], prompt[None].cuda())
    return om, h, wd, prompt


@pytest.mark.gpu
def test_tiny_steps_block_and_handoff(dg):
    om, h, wd, prompt = _setup(dg)
    n, vocab = M["canvas"], M["vocab"]
    assert dg.dg_get_length(h, 0) == W["prompt_len"]

    # oracle trajectory of block 0 (its cache grows by the hand-off at the end)
    o_tok, o_steps, trace = om.generate_block(0, seed=S["seed"], block=0, max_steps=S["max_steps"],
                                              schedule_steps=S["schedule_steps"], temperature=S["temperature"],
                                              stop_threshold=S["stop_threshold"])

    # 1) step by step through dg_denoise_step (the GPU follows its own outputs)
    canvas = torch.from_numpy(O.init_canvas(S["seed"], n, vocab, 0, 0).astype(np.int32)).cuda()[None]
    prev = None
    for t, ref in enumerate(trace, start=1):
        assert np.array_equal(to_np(canvas)[0], ref["canvas_in"]), f"canvas diverged before step {t}"
        logits = torch.zeros((1, n, vocab), device="cuda")
        outs = dict(x_hat=torch.zeros((1, n), dtype=torch.int32, device="cuda"),
                    pmax=torch.zeros((1, n), device="cuda"), entropy=torch.zeros((1, n), device="cuda"),
                    keep=torch.zeros((1, n), dtype=torch.int32, device="cuda"),
                    mean_entropy=torch.zeros(1, device="cuda"), stop=torch.zeros(1, dtype=torch.int32, device="cuda"),
                    experts_touched=torch.zeros(M["n_layers"], dtype=torch.int32, device="cuda"))
        sp = dg.sampler_params(temperature=S["temperature"], keep_k=O.linear_keep_count(n, t, S["schedule_steps"]),
                               stop_threshold=S["stop_threshold"], seed=S["seed"], block=0)
        dg.dg_denoise_step(h, [0], canvas, prev, t, sp, dg.step_out(**outs), logits_out=logits)
        dg.dg_synchronize(h)
        err = max_abs_rel(to_np(logits)[0], ref["logits"])
        assert err < 1e-4, f"step {t}: logits max-abs-rel {err}"
        check_decisions(to_np(outs["x_hat"])[0], ref["x_hat"], ref["sample_margin"], f"x_hat step {t}",
                        max_low_margin=0)
        assert np.allclose(to_np(outs["entropy"])[0], ref["H"], rtol=1e-4, atol=1e-5)
        if ref["keep_margin"] > 1e-5:
            assert np.array_equal(to_np(outs["keep"])[0].astype(bool), ref["keep"])
        assert bool(to_np(outs["stop"])[0]) == ref["stop"]
        touched = to_np(outs["experts_touched"])
        assert (touched >= 1).all() and (touched <= M["n_experts"]).all()
        if ref["stop"]:
            break
        prev = outs["x_hat"].clone()
    assert dg.dg_get_length(h, 0) == W["prompt_len"]      # steps do not advance the cache

    # 2) the whole block through dg_generate_block, then the hand-off
    out = torch.zeros((1, n), dtype=torch.int32, device="cuda")
    a = dg.block_args([0], S["max_steps"], S["schedule_steps"], temperature=S["temperature"],
                      stop_threshold=S["stop_threshold"], seed=S["seed"], block=0)
    steps = dg.dg_generate_block(h, a, out)
    assert steps == o_steps
    assert np.array_equal(to_np(out)[0], o_tok)
    assert dg.dg_get_length(h, 0) == W["prompt_len"] + n

    # 3) the appended K/V: the next block's first step sees the same cache
    canvas1 = O.init_canvas(S["seed"], n, vocab, 1, 0)
    ref_logits = om.denoise_forward(0, canvas1)
    logits = torch.zeros((1, n, vocab), device="cuda")
    sp = dg.sampler_params(temperature=1.0, keep_k=1, seed=S["seed"], block=1)
    c1 = torch.from_numpy(canvas1.astype(np.int32)).cuda()[None]
    dg.dg_denoise_step(h, [0], c1, None, 1, sp, dg.step_out(), logits_out=logits)
    dg.dg_synchronize(h)
    assert max_abs_rel(to_np(logits)[0], ref_logits) < 1e-4
    h.close()


@pytest.mark.gpu
def test_tiny_batch_of_two_requests_with_self_conditioning(dg):
    om, h, wd, prompt = _setup(dg)
    n, vocab = M["canvas"], M["vocab"]
    # request slot 1 gets a different, longer prompt
    prompt1 = synth.uniform_tokens(45, vocab, seed=77)
    dg.dg_prefill_prompt(h, [1], prompt1[None].cuda())
    om.encode_causal(1, prompt1.numpy())
    c = synth.uniform_tokens(n, vocab, seed=8, batch=2)
    prev = synth.uniform_tokens(n, vocab, seed=9, batch=2)
    logits = torch.zeros((2, n, vocab), device="cuda")
    hid = torch.zeros((2 * n, M["d_model"]), device="cuda")
    sp = dg.sampler_params(temperature=0.9, keep_k=5, seed=3, block=0)
    dg.dg_denoise_step(h, [1, 0], c.cuda(), prev.cuda(), 2, sp, dg.step_out(), logits_out=logits, hidden_out=hid)
    dg.dg_synchronize(h)
    for b, req in enumerate([1, 0]):
        ref, hidden = om.denoise_forward(req, c[b].numpy(), prev[b].numpy(), return_hidden=True)
        assert max_abs_rel(to_np(logits)[b], ref) < 1e-4
        assert max_abs_rel(to_np(hid)[b * n:(b + 1) * n], hidden) < 1e-4
    h.close()


@pytest.mark.gpu
def test_capacity_and_argument_errors_leave_state_unchanged(dg):
    om, h, wd, prompt = _setup(dg)
    big = torch.zeros((1, 128), dtype=torch.int32, device="cuda")
    with pytest.raises(dg.DgError) as e:
        dg.dg_prefill_prompt(h, [0], big)          # 32 + 128 > max_ctx 128
    assert e.value.code == dg.DG_ECAPACITY
    assert dg.dg_get_length(h, 0) == W["prompt_len"]
    with pytest.raises(dg.DgError) as e:
        dg.dg_prefill_prompt(h, [0, 0], big[:, :4].repeat(2, 1))
    assert e.value.code == dg.DG_EINVAL
    with pytest.raises(dg.DgError) as e:
        dg.dg_set_length(h, 0, 129)
    assert e.value.code == dg.DG_ECAPACITY
    h.close()
