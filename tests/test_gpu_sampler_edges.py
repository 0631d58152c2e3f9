"""Edge cases of the sampler on the GPU, through the C ABI, against closed forms.

- Uniform logits over the full 262144-token vocabulary make every statistic
  exact: each exp(z - max) is 1, every sum is an integer, u*V is exact. So
  pmax = 2^-18, H = ln 2^18, x_hat = floor(u V) with the Philox uniform u, and
  the keep set is decided by the index tie rule alone.
- keep_k = 0 re-noises every position; keep_k = N re-noises none.
- A one-token vocabulary (x_hat = 0, pmax = 1, H = 0, the stop fires), and a
  one-position canvas against the oracle.
- An empty batch is refused before anything is launched.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dg_oracle as O
from tests._util import check_decisions, to_np


def _handle(dg, B, vocab, n):
    return dg.dg_create(dict(vocab=vocab, canvas=n), None, dtype="fp32", max_batch=B, max_ctx=max(64, n))


def _run(dg, h, logits, req, step, sp, noalloc=False):
    B, n = logits.shape[0], logits.shape[1]
    dev = "cuda"
    outs = dict(x_hat=torch.full((B, n), -7, dtype=torch.int32, device=dev),
                pmax=torch.zeros((B, n), device=dev), entropy=torch.full((B, n), -1.0, device=dev),
                keep=torch.full((B, n), -1, dtype=torch.int32, device=dev),
                mean_entropy=torch.full((B,), -1.0, device=dev), stop=torch.full((B,), -1, dtype=torch.int32,
                                                                                 device=dev))
    canvas = torch.full((B, n), -1, dtype=torch.int32, device=dev)
    if noalloc:
        stream = torch.cuda.current_stream()
        dg.dg_sample_noalloc(logits, req, step, sp, canvas, dg.step_out(**outs), stream=stream)
        stream.synchronize()
    else:
        dg.dg_sample(h, logits, req, step, sp, canvas, dg.step_out(**outs))
        dg.dg_synchronize(h)
    outs["canvas"] = canvas
    return {k: to_np(v) for k, v in outs.items()}


@pytest.mark.gpu
def test_uniform_logits_full_vocab_are_exact(dg):
    n, V, k, seed, step, block = 256, 262144, 100, 9, 3, 2
    h = _handle(dg, 1, V, n)
    logits = torch.zeros((1, n, V), device="cuda")
    sp = dg.sampler_params(temperature=0.8, keep_k=k, stop_threshold=0.1, seed=seed, block=block)
    got = _run(dg, h, logits, [0], step, sp)
    h.close()
    words = O.sampler_words(seed, np.arange(n), step, block, 0)
    u = O.unit_uniform(words[:, 0])
    assert (got["pmax"][0] == np.float32(2.0 ** -18)).all()
    assert np.allclose(got["entropy"][0], math.log(V), rtol=1e-7, atol=0)
    assert np.array_equal(got["x_hat"][0], np.floor(u * V).astype(np.int64))
    # equal confidence everywhere: the k lowest positions are kept
    assert got["keep"][0].tolist() == [1] * k + [0] * (n - k)
    renoise = O.uniform_token(words[:, 1], V)
    assert np.array_equal(got["canvas"][0][:k], got["x_hat"][0][:k])
    assert np.array_equal(got["canvas"][0][k:], renoise[k:])
    assert abs(got["mean_entropy"][0] - math.log(V)) <= 1e-6 * math.log(V)
    assert got["stop"][0] == 0


@pytest.mark.gpu
@pytest.mark.parametrize("noalloc", [False, True])
def test_keep_none_and_keep_all(dg, noalloc):
    B, n, V = 2, 48, 4099                     # a vocabulary that is not a multiple of 4
    logits = torch.randn((B, n, V), generator=torch.Generator().manual_seed(41)).cuda()
    h = None if noalloc else _handle(dg, B, V, n)
    req = [1, 0]
    none = _run(dg, h, logits, req, 2, dg.sampler_params(temperature=1.0, keep_k=0, seed=4), noalloc)
    every = _run(dg, h, logits, req, 2, dg.sampler_params(temperature=1.0, keep_k=n, seed=4), noalloc)
    if h is not None:
        h.close()
    for b, r in enumerate(req):
        renoise = O.uniform_token(O.sampler_words(4, np.arange(n), 2, 0, r)[:, 1], V)
        assert (none["keep"][b] == 0).all() and np.array_equal(none["canvas"][b], renoise)
        assert (every["keep"][b] == 1).all() and np.array_equal(every["canvas"][b], every["x_hat"][b])
        # the keep rule does not touch the sample or the statistics
        assert np.array_equal(none["x_hat"][b], every["x_hat"][b])
        assert np.array_equal(none["entropy"][b], every["entropy"][b])


@pytest.mark.gpu
@pytest.mark.parametrize("temperature", [0.8, 0.0])
def test_one_token_vocabulary(dg, temperature):
    B, n = 2, 5
    logits = torch.randn((B, n, 1), generator=torch.Generator().manual_seed(43)).cuda()
    h = _handle(dg, B, 1, n)
    sp = dg.sampler_params(temperature=temperature, keep_k=2, stop_threshold=0.1, seed=3)
    got = _run(dg, h, logits, [0, 1], 1, sp)
    alt = _run(dg, None, logits, [0, 1], 1, sp, noalloc=True)
    h.close()
    for key in ("x_hat", "canvas", "keep", "stop"):
        assert np.array_equal(got[key], alt[key]), key
    assert (got["x_hat"] == 0).all() and (got["canvas"] == 0).all()
    assert (got["pmax"] == 1.0).all() and (got["entropy"] == 0.0).all()
    assert (got["mean_entropy"] == 0.0).all() and (got["stop"] == 1).all()
    assert got["keep"].sum(axis=1).tolist() == [2, 2]


@pytest.mark.gpu
def test_one_position_canvas(dg):
    B, n, V = 3, 1, 5000
    logits = torch.randn((B, n, V), generator=torch.Generator().manual_seed(45)) * 3.0
    h = _handle(dg, B, V, n)
    req = [2, 0, 1]
    sp = dg.sampler_params(temperature=0.9, keep_k=1, stop_threshold=50.0, seed=6, block=1)
    got = _run(dg, h, logits.cuda(), req, 4, sp)
    h.close()
    for b, r in enumerate(req):
        ref = O.sample_canvas(logits[b].numpy(), seed=6, step=4, block=1, req=r, temperature=0.9, logit_scale=1.0,
                              keep_k=1, stop_threshold=50.0)
        assert np.allclose(got["pmax"][b], ref["pmax"], rtol=1e-4, atol=1e-7)
        assert np.allclose(got["entropy"][b], ref["H"], rtol=1e-4, atol=1e-5)
        check_decisions(got["x_hat"][b], ref["x_hat"], ref["sample_margin"], "x_hat", max_low_margin=0)
        assert got["keep"][b].tolist() == [1] and got["canvas"][b].tolist() == got["x_hat"][b].tolist()
        assert abs(got["mean_entropy"][b] - got["entropy"][b][0]) <= 1e-6 * max(1.0, got["entropy"][b][0])
        assert got["stop"][b] == int(ref["stop"])


@pytest.mark.gpu
def test_empty_batch_is_refused(dg):
    h = _handle(dg, 2, 1000, 8)
    logits = torch.zeros((1, 8, 1000), device="cuda")
    canvas = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="batch 0"):
        dg.dg_sample(h, logits, [], 1, dg.sampler_params(keep_k=1), canvas, dg.step_out())
    h.close()
