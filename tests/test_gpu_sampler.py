"""Sampler-only workload: logits [B, 256, 262144] = Gumbel + a peak of height
U(0,12) at a random token; temperature 0.8; keep k in {64, 128, 192}; stop 0.1.
The GPU sampler (dg_sample, through the C ABI) against the oracle on the same
logits and Philox counters."""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import check_decisions, to_np

W = synth.WORKLOADS["sampler"]


def _handle(dg, B, vocab=W["vocab"], n=W["canvas"]):
    return dg.dg_create(dict(vocab=vocab, canvas=n), None, dtype="fp32", max_batch=B, max_ctx=max(64, n))


def _run(dg, h, logits, req, step, sp):
    B, n = logits.shape[0], logits.shape[1]
    dev = logits.device
    outs = dict(x_hat=torch.zeros((B, n), dtype=torch.int32, device=dev),
                pmax=torch.zeros((B, n), device=dev), entropy=torch.zeros((B, n), device=dev),
                keep=torch.zeros((B, n), dtype=torch.int32, device=dev),
                mean_entropy=torch.zeros(B, device=dev), stop=torch.zeros(B, dtype=torch.int32, device=dev))
    canvas = torch.full((B, n), -1, dtype=torch.int32, device=dev)
    dg.dg_sample(h, logits, req, step, sp, canvas, dg.step_out(**outs))
    dg.dg_synchronize(h)
    outs["canvas"] = canvas
    return {k: to_np(v) for k, v in outs.items()}


def _compare(got, ref, b):
    assert np.allclose(got["pmax"][b], ref["pmax"], rtol=1e-4, atol=1e-7)
    assert np.allclose(got["entropy"][b], ref["H"], rtol=1e-4, atol=1e-5)
    low = check_decisions(got["x_hat"][b], ref["x_hat"], ref["sample_margin"], "x_hat")
    if ref["keep_margin"] > 1e-5:
        assert np.array_equal(got["keep"][b].astype(bool), ref["keep"])
        same = got["x_hat"][b] == ref["x_hat"]     # low-margin samples may differ
        assert np.array_equal(got["canvas"][b][same], ref["x_new"][same])
    # whatever the keep set, re-noised positions hold the Philox token
    rn = got["keep"][b] == 0
    assert np.array_equal(got["canvas"][b][rn], ref["renoise"][rn])
    assert np.array_equal(got["canvas"][b][~rn], got["x_hat"][b][~rn])
    assert abs(got["mean_entropy"][b] - ref["mean_H"]) <= 1e-4 * max(1.0, abs(ref["mean_H"]))
    if ref["stop_margin"] > 1e-5:
        assert bool(got["stop"][b]) == ref["stop"]
    return low


@pytest.mark.gpu
@pytest.mark.parametrize("k", W["keep"])
def test_sampler_batch1_full_vocab(dg, k):
    logits, _, _ = synth.peaked_logits(1, W["canvas"], W["vocab"], seed=W["seed"] + k, peak_max=W["peak_max"])
    h = _handle(dg, 1)
    sp = dg.sampler_params(temperature=W["temperature"], keep_k=k, stop_threshold=W["stop_threshold"],
                           seed=123, block=2)
    got = _run(dg, h, logits.cuda(), [0], 3, sp)
    ref = O.sample_canvas(logits[0].numpy(), seed=123, step=3, block=2, req=0, temperature=W["temperature"],
                          logit_scale=1.0, keep_k=k, stop_threshold=W["stop_threshold"])
    low = _compare(got, ref, 0)
    assert low <= 2
    h.close()


@pytest.mark.gpu
def test_sampler_zero_temperature_is_argmax(dg):
    logits, _, _ = synth.peaked_logits(1, W["canvas"], W["vocab"], seed=7)
    logits[0, 5, :] = 0.0                       # all tied: argmax = 0, H = log V
    logits[0, 6, 17] = logits[0, 6, 99] = 1e3   # a two-way tie
    h = _handle(dg, 1)
    sp = dg.sampler_params(temperature=0.0, keep_k=100, stop_threshold=0.1, seed=1)
    got = _run(dg, h, logits.cuda(), [0], 1, sp)
    ref = O.sample_canvas(logits[0].numpy(), seed=1, step=1, block=0, req=0, temperature=0.0, logit_scale=1.0,
                          keep_k=100, stop_threshold=0.1)
    assert np.array_equal(got["x_hat"][0], logits[0].argmax(-1).numpy())
    assert got["x_hat"][0, 6] == 17
    assert np.allclose(got["pmax"][0], ref["pmax"]) and np.allclose(got["entropy"][0], ref["H"], atol=1e-6)
    assert np.array_equal(got["keep"][0].astype(bool), ref["keep"])
    assert np.array_equal(got["canvas"][0], ref["x_new"])
    h.close()


@pytest.mark.gpu
def test_sampler_small_vocab_ragged_chunks(dg):
    # vocab not a multiple of 4 or of the 4096-logit chunk, canvas not a multiple of 32
    g = torch.Generator().manual_seed(5)
    B, n, vocab = 3, 37, 5001
    logits = torch.randn((B, n, vocab), generator=g) * 3
    h = _handle(dg, B, vocab=vocab, n=n)
    sp = dg.sampler_params(temperature=1.3, logit_scale=0.7, keep_k=11, stop_threshold=5.0, seed=99, block=4)
    got = _run(dg, h, logits.cuda(), [2, 0, 1], 6, sp)
    for b, req in enumerate([2, 0, 1]):
        ref = O.sample_canvas(logits[b].numpy(), seed=99, step=6, block=4, req=req, temperature=1.3,
                              logit_scale=0.7, keep_k=11, stop_threshold=5.0)
        _compare(got, ref, b)
    h.close()


@pytest.mark.gpu
@pytest.mark.parametrize("B,k", [(16, 128), (64, 192)])
def test_sampler_large_batch_sampled_canvases(dg, B, k):
    g = torch.Generator(device="cuda").manual_seed(W["seed"] * 100 + B)
    # generate on the device in chunks: [B, 256, 262144] fp32 (17 GB at B = 64)
    logits = torch.empty((B, W["canvas"], W["vocab"]), device="cuda")
    for b in range(B):
        u = torch.rand((W["canvas"], W["vocab"]), generator=g, device="cuda").clamp_(min=1e-30)
        logits[b] = -torch.log(-torch.log(u))
        r = torch.randint(0, W["vocab"], (W["canvas"],), generator=g, device="cuda")
        hgt = torch.rand((W["canvas"],), generator=g, device="cuda") * W["peak_max"]
        logits[b].scatter_add_(1, r[:, None], hgt[:, None])
    req = list(range(B))
    h = _handle(dg, B)
    sp = dg.sampler_params(temperature=W["temperature"], keep_k=k, stop_threshold=W["stop_threshold"], seed=5)
    got = _run(dg, h, logits, req, 2, sp)
    for b in (0, B - 1):
        ref = O.sample_canvas(logits[b].cpu().numpy(), seed=5, step=2, block=0, req=b,
                              temperature=W["temperature"], logit_scale=1.0, keep_k=k,
                              stop_threshold=W["stop_threshold"])
        _compare(got, ref, b)
    del logits
    torch.cuda.empty_cache()
    h.close()


@pytest.mark.gpu
def test_sampler_rejects_unaligned_logits(dg):
    """Pass 1 reads the logits with 16-byte loads: an unaligned pointer is refused on the host."""
    n, V = 32, 1024
    h = _handle(dg, 1, vocab=V, n=n)
    buf = torch.zeros(n * V + 4, device="cuda")
    canvas = torch.zeros((1, n), dtype=torch.int32, device="cuda")
    sp = dg.sampler_params(temperature=1.0, keep_k=4)
    with pytest.raises(dg.DgError) as ei:
        dg.dg_sample(h, buf[1:], [0], 1, sp, canvas, dg.step_out())
    assert ei.value.code == 1 and "aligned" in str(ei.value)
    dg.dg_sample(h, buf[4:], [0], 1, sp, canvas, dg.step_out())   # 16-byte offset is fine
    dg.dg_synchronize(h)
    h.close()
