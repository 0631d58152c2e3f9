"""The page's sampler variants on the GPU, against the oracle.

- Entropy-budget keep (dg_sample, dg_sample_noalloc): the sampler workload's
  peaked logits (256 x 262144, T 0.8) at budgets 0, the page's 0.1, 50 nats
  and one that keeps everything; a batch of three canvases over a ragged
  5001-token vocabulary.  The keep set must equal the oracle's budget set of
  the GPU's own entropies exactly (the running sums are fp64 on both sides),
  and the oracle's set of its own entropies where the crossing sum is not
  within 1e-3 of the budget.
- Temperature anneal and the budget keep in the block loop (tiny fp32 model):
  each step checked against the oracle from the GPU's own canvas, then
  dg_generate_block must reproduce that trajectory token for token.
- Two-round stop: the sampler on peaked logits over four rounds (argmax
  unchanged, one position changed, a previous round above the threshold)
  through dg_sample and dg_sample_noalloc; the argmax output against the
  oracle's; in the tiny model's block (T = 0, every position kept) step by
  step and through dg_generate_block.
- Argument errors: unknown keep_mode and stop_mode, bad budgets, bad anneal ends.
"""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import check_decisions, max_abs_rel, to_np

SW = synth.WORKLOADS["sampler"]
TW = synth.WORKLOADS["tiny_fp32"]


def _outs(B, n, argmax=False):
    dev = "cuda"
    o = dict(x_hat=torch.zeros((B, n), dtype=torch.int32, device=dev),
             pmax=torch.zeros((B, n), device=dev), entropy=torch.zeros((B, n), device=dev),
             keep=torch.zeros((B, n), dtype=torch.int32, device=dev),
             mean_entropy=torch.zeros(B, device=dev), stop=torch.zeros(B, dtype=torch.int32, device=dev))
    if argmax:
        o["argmax"] = torch.full((B, n), -1, dtype=torch.int32, device=dev)
    return o


def _sample(dg, logits, req, step, sp, noalloc=False, argmax=False, keep_tensors=False):
    B, n, V = logits.shape
    outs = _outs(B, n, argmax)
    canvas = torch.full((B, n), -1, dtype=torch.int32, device="cuda")
    if noalloc:
        stream = torch.cuda.current_stream()
        dg.dg_sample_noalloc(logits, req, step, sp, canvas, dg.step_out(**outs), stream=stream)
        stream.synchronize()
    else:
        h = dg.dg_create(dict(vocab=V, canvas=n), None, dtype="fp32", max_batch=max(req) + 1, max_ctx=max(64, n))
        dg.dg_sample(h, logits, req, step, sp, canvas, dg.step_out(**outs))
        dg.dg_synchronize(h)
        h.close()
    outs["canvas"] = canvas
    if keep_tensors:
        return outs
    return {k: to_np(v) for k, v in outs.items()}


def _oracle(lg, *, seed, step, block, req, temperature):
    """The oracle's statistics, samples and re-noise tokens of one canvas (the keep rule does not touch them)."""
    return O.sample_canvas(lg, seed=seed, step=step, block=block, req=req, temperature=temperature,
                           logit_scale=1.0, keep_k=0, stop_threshold=-1.0)


def _check_budget_canvas(got, b, ref, budget):
    ref = dict(ref)
    ref["keep"], ref["keep_margin"] = O.keep_entropy_budget(ref["H"], budget)
    assert np.allclose(got["entropy"][b], ref["H"], rtol=1e-4, atol=1e-5)
    check_decisions(got["x_hat"][b], ref["x_hat"], ref["sample_margin"], "x_hat", max_low_margin=2)
    keep = got["keep"][b].astype(bool)
    # the budget set of the GPU's own entropies: exact up to fp64 summation order
    own, own_margin = O.keep_entropy_budget(got["entropy"][b].astype(np.float64), budget)
    if own_margin > 1e-9:
        assert np.array_equal(keep, own)
    # ... and the oracle's own set wherever fp32 entropies cannot move the crossing
    if ref["keep_margin"] > 1e-3:
        assert np.array_equal(keep, ref["keep"])
    assert np.array_equal(got["canvas"][b][keep], got["x_hat"][b][keep])
    assert np.array_equal(got["canvas"][b][~keep], ref["renoise"][~keep])
    return int(keep.sum())


@pytest.mark.gpu
def test_entropy_budget_keep_full_vocab(dg):
    n, V = SW["canvas"], SW["vocab"]
    logits, _, _ = synth.peaked_logits(1, n, V, seed=SW["seed"] + 501, peak_max=SW["peak_max"])
    ref = _oracle(logits[0].numpy(), seed=41, step=2, block=3, req=0, temperature=SW["temperature"])
    g = logits.cuda()
    counts = []
    for budget in (0.0, 0.1, 50.0, 1e30):
        b32 = float(np.float32(budget))
        sp = dg.sampler_params(temperature=SW["temperature"], keep_k=0, seed=41, block=3, entropy_budget=b32)
        got = _sample(dg, g, [0], 2, sp)
        counts.append(_check_budget_canvas(got, 0, ref, b32))
        # the no-allocation entry point runs the same kernels
        alt = _sample(dg, g, [0], 2, sp, noalloc=True)
        for k in ("keep", "canvas", "x_hat"):
            assert np.array_equal(alt[k], got[k]), k
    assert counts[0] == 1                          # a zero budget locks only the most certain position
    assert counts[-1] == n                         # an unbounded budget keeps every position
    assert counts == sorted(counts)                # a larger budget never keeps fewer


@pytest.mark.gpu
def test_entropy_budget_keep_batch_ragged_vocab(dg):
    B, n, V = 3, 37, 5001
    gen = torch.Generator().manual_seed(17)
    scale = torch.rand((B, n, 1), generator=gen) * 8.0      # from flat to sharply peaked rows
    logits = torch.randn((B, n, V), generator=gen) * scale
    req = [2, 0, 1]
    sp = dg.sampler_params(temperature=0.7, keep_k=0, stop_threshold=3.0, seed=9, block=1, entropy_budget=20.0)
    got = _sample(dg, logits.cuda(), req, 5, sp)
    for b, r in enumerate(req):
        _check_budget_canvas(got, b, _oracle(logits[b].numpy(), seed=9, step=5, block=1, req=r, temperature=0.7),
                             20.0)
        mh = float(np.mean(got["entropy"][b].astype(np.float64)))
        assert abs(got["mean_entropy"][b] - mh) <= 1e-5 * max(1.0, mh)


def _tiny(dg):
    M = TW["model"]
    w = synth.make_weights(M, seed=TW["seed"], dtype="fp32", router_bias=TW["router_bias"])
    prompt = synth.uniform_tokens(TW["prompt_len"], M["vocab"], seed=TW["seed"] + 100)
    om = O.OracleModel(dict(M), synth.to_numpy_weights(w))
    om.encode_causal(0, prompt.numpy())
    wd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in w.items() if k != "layers"}
    wd["layers"] = [{k: (None if v is None else v.cuda()) for k, v in L.items()} for L in w["layers"]]
    h = dg.dg_create(M, wd, dtype="fp32", max_batch=1, max_ctx=128)
    dg.dg_prefill_prompt(h, [0], prompt[None].cuda())
    return om, h, wd


@pytest.mark.gpu
def test_block_with_anneal_and_entropy_budget(dg):
    om, h, wd = _tiny(dg)
    M, S = TW["model"], TW["sampler"]
    n, vocab, steps_max = M["canvas"], M["vocab"], S["max_steps"]
    t0, t1 = float(np.float32(0.8)), float(np.float32(0.4))
    budget = 20.0
    seed, block = S["seed"], 0
    # 1) step by step: each step's inputs are the GPU's own, checked against the oracle
    canvas = torch.from_numpy(O.init_canvas(seed, n, vocab, block, 0).astype(np.int32)).cuda()[None]
    prev = None
    traj = []
    for t in range(1, steps_max + 1):
        temp = float(np.float32(O.anneal_temperature(t, steps_max, t0, t1)))
        c_in = to_np(canvas)[0].copy()
        logits = torch.zeros((1, n, vocab), device="cuda")
        outs = _outs(1, n)
        sp = dg.sampler_params(temperature=temp, keep_k=0, stop_threshold=S["stop_threshold"], seed=seed,
                               block=block, entropy_budget=budget)
        dg.dg_denoise_step(h, [0], canvas, prev, t, sp, dg.step_out(**outs), logits_out=logits)
        dg.dg_synchronize(h)
        got = {k: to_np(v) for k, v in outs.items()}
        ref = om.denoise_step(0, c_in, None if prev is None else to_np(prev)[0], step=t, block=block, seed=seed,
                              temperature=temp, logit_scale=1.0, keep_k=0, stop_threshold=S["stop_threshold"],
                              keep_budget=budget)
        assert max_abs_rel(to_np(logits)[0], ref["logits"]) < 1e-4
        got["canvas"] = to_np(canvas)
        _check_budget_canvas(got, 0, ref, budget)
        if ref["stop_margin"] > 1e-5:
            assert bool(got["stop"][0]) == ref["stop"]
        traj.append(got)
        if got["stop"][0] or t == steps_max:
            break
        prev = outs["x_hat"].clone()
    # 2) the block loop anneals and keeps the same way: the same trajectory, token for token
    a = dg.block_args([0], steps_max, S["schedule_steps"], temperature=t0, stop_threshold=S["stop_threshold"],
                      seed=seed, block=block, entropy_budget=budget, temperature_end=t1)
    out = torch.zeros((1, n), dtype=torch.int32, device="cuda")
    steps = dg.dg_generate_block(h, a, out)
    assert steps == len(traj)
    assert np.array_equal(to_np(out)[0], traj[-1]["x_hat"][0])
    assert dg.dg_get_length(h, 0) == TW["prompt_len"] + n
    h.close()


@pytest.mark.gpu
def test_variant_argument_errors(dg):
    n, V = 16, 1000
    h = dg.dg_create(dict(vocab=V, canvas=n), None, dtype="fp32", max_batch=1, max_ctx=64)
    logits = torch.zeros((1, n, V), device="cuda")
    canvas = torch.zeros((1, n), dtype=torch.int32, device="cuda")
    bad = dg.sampler_params(temperature=1.0, keep_k=1)
    bad.keep_mode = 3
    with pytest.raises(RuntimeError, match="keep_mode"):
        dg.dg_sample(h, logits, [0], 1, bad, canvas, dg.step_out())
    for budget in (-1.0, float("nan")):
        with pytest.raises(RuntimeError, match="budget"):
            dg.dg_sample(h, logits, [0], 1, dg.sampler_params(entropy_budget=budget), canvas, dg.step_out())
    bad = dg.sampler_params(temperature=1.0, keep_k=1)
    bad.stop_mode = 2
    with pytest.raises(RuntimeError, match="stop_mode"):
        dg.dg_sample(h, logits, [0], 1, bad, canvas, dg.step_out())
    h.close()
    om, ht, wd = _tiny(dg)
    S = TW["sampler"]
    out = torch.zeros((1, TW["model"]["canvas"]), dtype=torch.int32, device="cuda")
    bad_stop = dg.block_args([0], 2, 2, seed=S["seed"])
    bad_stop.stop_mode = 5
    for kw in (dict(temperature=0.8, temperature_end=0.0), dict(temperature=0.0, temperature_end=0.4),
               dict(temperature=0.8, entropy_budget=-2.0), None):
        a = bad_stop if kw is None else dg.block_args([0], 2, 2, seed=S["seed"], **kw)
        with pytest.raises(RuntimeError):
            dg.dg_generate_block(ht, a, out)
        assert dg.dg_get_length(ht, 0) == TW["prompt_len"]     # refused before anything ran
    ht.close()


@pytest.mark.gpu
@pytest.mark.parametrize("noalloc", [False, True])
def test_two_round_stop_sampler(dg, noalloc):
    B, n, V, tau = 2, 64, 5000, 0.005
    gen = torch.Generator().manual_seed(31)
    base = torch.randn((B, n, V), generator=gen)
    peak = torch.randint(0, V, (B, n), generator=gen)
    l1 = base.clone()
    l1.scatter_(2, peak[..., None], 30.0)                    # H ~ 1e-8 nats per position
    l2 = l1 * 1.01                                           # the same argmax
    l3 = l2.clone()
    l3[1, 7] = base[1, 7]
    l3[1, 7, (int(peak[1, 7]) + 1) % V] = 30.0              # canvas 1 changes one position's argmax
    rounds = [(l1, None, None), (l2, "prev", None), (l3, "prev", None), (l2, "prev", 1.0)]
    want_stop = [[0, 0], [1, 1], [1, 0], [0, 0]]
    prev = None
    for r, ((lg, use_prev, prev_h), want) in enumerate(zip(rounds, want_stop)):
        pa = pm = None
        if use_prev:
            pa = prev["argmax"]
            pm = prev["mean_entropy"] if prev_h is None else torch.full((B,), prev_h, device="cuda")
        sp = dg.sampler_params(temperature=1.0, keep_k=n, stop_threshold=tau, seed=5, block=0,
                               two_round_stop=True, prev_argmax=pa, prev_mean_entropy=pm)
        outs = _sample(dg, lg.cuda(), [0, 1], r + 1, sp, noalloc=noalloc, argmax=True, keep_tensors=True)
        got = {k: to_np(v) for k, v in outs.items()}
        for b in range(B):
            ref = _oracle(lg[b].numpy(), seed=5, step=r + 1, block=0, req=b, temperature=1.0)
            check_decisions(got["argmax"][b], ref["argmax"], ref["argmax_margin"], "argmax", thr=1e-6,
                            max_low_margin=0)
            assert got["mean_entropy"][b] < tau
            # the stop is the oracle's rule on this round's and the previous round's GPU outputs
            want_rule = O.stop_two_rounds(None if pm is None else float(to_np(pm)[b]), float(got["mean_entropy"][b]),
                                          None if pa is None else to_np(pa)[b], got["argmax"][b], tau=tau)
            assert bool(got["stop"][b]) == want_rule
        assert got["stop"].tolist() == want, f"round {r + 1}"
        prev = outs


@pytest.mark.gpu
def test_argmax_output_at_zero_temperature_is_x_hat(dg):
    B, n, V = 2, 40, 3001
    logits = torch.randn((B, n, V), generator=torch.Generator().manual_seed(33))
    sp = dg.sampler_params(temperature=0.0, keep_k=5, seed=1)
    got = _sample(dg, logits.cuda(), [0, 1], 1, sp, argmax=True)
    assert np.array_equal(got["argmax"], got["x_hat"])
    assert np.array_equal(got["argmax"], logits.argmax(-1).numpy())


@pytest.mark.gpu
def test_block_with_two_round_stop(dg):
    om, h, wd = _tiny(dg)
    M, S = TW["model"], TW["sampler"]
    n, vocab, steps_max, tau = M["canvas"], M["vocab"], 8, 0.1
    seed, block = S["seed"], 0
    # 1) step by step at T = 0 with every position kept: the canvas becomes the argmax
    canvas = torch.from_numpy(O.init_canvas(seed, n, vocab, block, 0).astype(np.int32)).cuda()[None]
    prev_x = prev = None
    traj = []
    for t in range(1, steps_max + 1):
        c_in = to_np(canvas)[0].copy()
        logits = torch.zeros((1, n, vocab), device="cuda")
        outs = _outs(1, n, argmax=True)
        sp = dg.sampler_params(temperature=0.0, keep_k=n, stop_threshold=tau, seed=seed, block=block,
                               two_round_stop=True, prev_argmax=None if prev is None else prev["argmax"],
                               prev_mean_entropy=None if prev is None else prev["mean_entropy"])
        dg.dg_denoise_step(h, [0], canvas, prev_x, t, sp, dg.step_out(**outs), logits_out=logits)
        dg.dg_synchronize(h)
        got = {k: to_np(v) for k, v in outs.items()}
        ref_logits = om.denoise_forward(0, c_in, None if prev_x is None else to_np(prev_x)[0])
        assert max_abs_rel(to_np(logits)[0], ref_logits) < 1e-4
        assert np.array_equal(got["argmax"][0], got["x_hat"][0])
        ref = _oracle(to_np(logits)[0], seed=seed, step=t, block=block, req=0, temperature=0.0)
        assert np.array_equal(got["argmax"][0], ref["argmax"])
        want = O.stop_two_rounds(None if prev is None else float(to_np(prev["mean_entropy"])[0]),
                                 float(got["mean_entropy"][0]), None if prev is None else to_np(prev["argmax"])[0],
                                 got["argmax"][0], tau=tau)
        assert bool(got["stop"][0]) == want
        traj.append(got)
        if got["stop"][0] or t == steps_max:
            break
        prev, prev_x = outs, outs["x_hat"]
    # 2) the block loop keeps the previous round itself: the same trajectory
    a = dg.block_args([0], steps_max, 1, temperature=0.0, stop_threshold=tau, seed=seed, block=block,
                      two_round_stop=True)
    out = torch.zeros((1, n), dtype=torch.int32, device="cuda")
    steps = dg.dg_generate_block(h, a, out)
    assert steps == len(traj)
    assert np.array_equal(to_np(out)[0], traj[-1]["x_hat"][0])
    h.close()
