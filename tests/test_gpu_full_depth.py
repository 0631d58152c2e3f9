"""The full-size workloads, in the handle configuration bench.py times.

- full_b1: 30 full-width layers, an 8192-token prompt, one 256-token canvas;
  up to 48 steps, linear keep over 48, stop at 0.1 nats, logit scale 1.5^(t-1).
- full_b16: 16 requests with 4096-token prompts, 4 blocks of 12 fixed steps.

A float64 pass through 30 layers is too slow for a test, so full depth is
checked on sampled outputs the oracle computes one by one, and by properties
that hold at any size.  (One full-width layer is compared whole in
test_gpu_layer.py.)

- The sampler's statistics and its Philox inverse-CDF decision, on sampled
  positions of the GPU's own logits.
- The final norm + tied LM head, on sampled rows (and vocabulary columns) of the GPU's own final
  hidden state.
- Keep count and keep set; kept positions hold x_hat and the others the Philox
  re-noise token; the mean entropy and the stop flag.
- Determinism of whole blocks, and the KV length after each hand-off.
- Layer by layer at layers 0, 14 and 29: the step records the residual stream
  entering and leaving the layer and the router's experts; the oracle runs the
  same layer on the GPU's own input and the request's cache as the GPU holds
  it (read back with dg_get_kv), on the canvas step of full_b1 (cache 8192)
  and of full_b16 (cache 4096, and 4352 after one hand-off).
"""
import gc

import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from tests._util import check_decisions, max_abs_rel, to_np

TOL_BF16 = 2e-2
ROWS = [0, 1, 77, 128, 200, 255]        # sampled canvas positions
N_VOCAB_COLS = 4096                     # sampled LM-head columns per row


def _setup(dg, name):
    W = synth.WORKLOADS[name]
    M, B, n, P0 = W["model"], W["batch"], W["model"]["canvas"], W["prompt_len"]
    blocks = W.get("blocks", 1)
    max_ctx = ((P0 + blocks * n + 63) // 64) * 64
    max_tokens = max(B * n, min(8192, B * P0))
    w = synth.make_weights(M, seed=W["seed"], dtype="bf16", router_bias=True, device="cuda")
    h = dg.dg_create(M, w, dtype="bf16", max_batch=B, max_ctx=max_ctx, max_tokens=max_tokens)
    prompt = synth.uniform_tokens(P0, M["vocab"], seed=W["seed"] + 1, batch=B, device="cuda")
    dg.dg_prefill_prompt(h, list(range(B)), prompt)
    dg.dg_synchronize(h)
    return W, w, h


def _release(h, w):
    h.close()
    del w
    gc.collect()
    torch.cuda.empty_cache()


def _check_step(dg, W, w, h, req, step, block, temperature, scale, keep_k, stop, check=None):
    """One explicit denoise step from the Philox initial canvas, checked on
    sampled positions of the requests in `check` (default: all)."""
    M, n, V = W["model"], W["model"]["canvas"], W["model"]["vocab"]
    B = len(req)
    seed = W["sampler"]["seed"]
    canvas0 = np.stack([O.init_canvas(seed, n, V, block, r) for r in req]).astype(np.int32)
    canvas = torch.from_numpy(canvas0).cuda()
    outs = dict(x_hat=torch.zeros((B, n), dtype=torch.int32, device="cuda"),
                pmax=torch.zeros((B, n), device="cuda"), entropy=torch.zeros((B, n), device="cuda"),
                keep=torch.zeros((B, n), dtype=torch.int32, device="cuda"),
                mean_entropy=torch.zeros(B, device="cuda"), stop=torch.zeros(B, dtype=torch.int32, device="cuda"))
    logits = torch.empty((B, n, V), device="cuda")
    hidden = torch.empty((B * n, M["d_model"]), device="cuda")
    sp = dg.sampler_params(temperature=temperature, logit_scale=scale, keep_k=keep_k, stop_threshold=stop,
                           seed=seed, block=block)
    dg.dg_denoise_step(h, req, canvas, None, step, sp, dg.step_out(**outs), logits_out=logits, hidden_out=hidden)
    dg.dg_synchronize(h)
    got = {k: to_np(v) for k, v in outs.items()}
    got_canvas = to_np(canvas)
    fn = to_np(w["final_norm"]).astype(np.float64)
    cols = np.sort(np.random.default_rng(step * 100 + block).choice(V, N_VOCAB_COLS, replace=False))
    emb_cols = to_np(w["embed"][torch.from_numpy(cols).cuda()].float()).astype(np.float64)
    for bi, r in enumerate(req):
        if check is not None and r not in check:
            continue
        lg = to_np(logits[bi, ROWS]).astype(np.float64)
        # final norm + tied LM head on the GPU's own hidden rows, on sampled vocabulary columns
        hid = to_np(hidden[bi * n + torch.tensor(ROWS)]).astype(np.float64)
        x = O.rms_norm(hid, fn, M["rms_eps"])
        assert max_abs_rel(lg[:, cols], x @ emb_cols.T) < TOL_BF16
        # sampler statistics and the inverse-CDF decision on the GPU's own logits
        words = O.sampler_words(seed, np.array(ROWS), step, block, r)
        u = O.unit_uniform(words[:, 0])
        xh, marg = [], []
        for k, row in enumerate(ROWS):
            st = O.position_stats(lg[k], temperature, scale)
            assert abs(got["pmax"][bi, row] - st["pmax"]) <= 1e-4 * st["pmax"] + 1e-7
            assert abs(got["entropy"][bi, row] - st["H"]) <= 1e-4 * max(1.0, st["H"])
            j, mg = O.inverse_cdf(st["e"], st["S"], u[k])
            xh.append(j)
            marg.append(mg)
        low = check_decisions(got["x_hat"][bi, ROWS], np.array(xh), np.array(marg), "x_hat")
        assert low <= 1
        # keep set, re-noise and stop, from the GPU's own statistics
        keep = got["keep"][bi].astype(bool)
        assert keep.sum() == keep_k
        ref_keep, kmargin = O.keep_set(got["pmax"][bi], keep_k)
        if kmargin > 1e-6:
            assert np.array_equal(keep, ref_keep)
        renoise = O.uniform_token(O.sampler_words(seed, np.arange(n), step, block, r)[:, 1], V)
        assert np.array_equal(got_canvas[bi][keep], got["x_hat"][bi][keep])
        assert np.array_equal(got_canvas[bi][~keep], renoise[~keep])
        mh = float(np.mean(got["entropy"][bi].astype(np.float64)))
        assert abs(got["mean_entropy"][bi] - mh) <= 1e-5 * max(1.0, mh)
        if stop >= 0 and abs(mh - stop) > 1e-5:
            assert bool(got["stop"][bi]) == (mh < stop)
    return got


PIN_LAYERS = (0, 14, 29)
ROUTER_MARGIN = 0.02      # router decisions closer than this are rounding-order ties (bf16 router input)


class _Experts:
    """One layer's stacked expert matrix [E, out, in] on the device, handed to
    the oracle one expert at a time (as float32 numpy, exact for bf16)."""

    def __init__(self, t):
        self.t = t
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            self.cache[e] = to_np(self.t[e].float())
        return self.cache[e]


def _oracle_layer_weights(w, li):
    L = w["layers"][li]
    out = {k: (None if v is None else to_np(v.float())) for k, v in L.items()
           if k not in ("w_gate", "w_up", "w_down")}
    for k in ("w_gate", "w_up", "w_down"):
        out[k] = _Experts(L[k])
    return out


def _layer_pins(dg, W, w, h, req, block, check, layers=PIN_LAYERS):
    """One canvas step per pinned layer, recording that layer; each request in
    `check` is compared with the oracle's layer on the GPU's input.  Returns the
    fraction of checked tokens excluded as router near-ties."""
    M = W["model"]
    n, d, k = M["canvas"], M["d_model"], M["top_k"]
    B = len(req)
    seed = W["sampler"]["seed"]
    canvas0 = np.stack([O.init_canvas(seed, n, M["vocab"], block, r) for r in req]).astype(np.int32)
    excluded, total = 0, 0
    for li in layers:
        hin = torch.empty((B * n, d), device="cuda")
        hout = torch.empty((B * n, d), device="cuda")
        ids = torch.empty((B * n, k), dtype=torch.int32, device="cuda")
        wts = torch.empty((B * n, k), device="cuda")
        sp = dg.sampler_params(temperature=1.0, keep_k=n // 2, seed=seed, block=block)
        dg.dg_denoise_step(h, req, torch.from_numpy(canvas0).cuda(), None, 1, sp, dg.step_out(),
                           dump=dg.layer_dump(li, hin, hout, ids, wts))
        dg.dg_synchronize(h)
        om = O.OracleModel(dict(M), {"layers": {li: _oracle_layer_weights(w, li)}})
        for bi, r in enumerate(req):
            if r not in check:
                continue
            P = dg.dg_get_length(h, r)
            kc = torch.empty((M["n_kv_heads"], P, M["head_dim"]), dtype=torch.bfloat16, device="cuda")
            vc = torch.empty_like(kc)
            dg.dg_get_kv(h, r, li, kc, vc)
            dg.dg_synchronize(h)
            om.set_kv(r, li, to_np(kc.float()), to_np(vc.float()))
            rows = slice(bi * n, (bi + 1) * n)
            x_in = to_np(hin[rows]).astype(np.float64)
            tr = {}
            ref, _, _ = om.layer(x_in, li, r, P + np.arange(n), causal=False, trace=tr)
            got = to_np(hout[rows]).astype(np.float64)
            gids = to_np(ids[rows])
            same = np.array([set(a) == set(b) for a, b in zip(gids.tolist(), tr["router_ids"].tolist())])
            # a token routed differently must be a near-tie of the oracle's router
            assert (tr["router_margin"][~same] < ROUTER_MARGIN).all(), \
                f"layer {li} req {r}: experts differ at margins {tr['router_margin'][~same]}"
            excluded += int((~same).sum())
            total += n
            err = float(np.max(np.abs(got[same] - ref[same])) / np.max(np.abs(ref)))
            assert err < TOL_BF16, f"layer {li} req {r}: output max-abs-rel {err}"
            # the layer's own contribution, out - in (the input is shared, so this isolates the layer)
            dref = ref - x_in
            derr = float(np.max(np.abs((got - x_in)[same] - dref[same])) / np.max(np.abs(dref)))
            assert derr < TOL_BF16, f"layer {li} req {r}: layer-delta max-abs-rel {derr}"
            gw = to_np(wts[rows])
            wmap = [dict(zip(a, b)) for a, b in zip(gids.tolist(), gw.tolist())]
            _, wref, _, _ = O.router(tr["moe_in"], om.weights["layers"][li]["router_w"],
                                     om.weights["layers"][li]["router_b"], k)
            for t in np.nonzero(same)[0][:64]:
                for e, wv in zip(tr["router_ids"][t], wref[t]):
                    assert abs(wmap[t][int(e)] - wv) < 2e-2 * max(wv, 1e-3) + 1e-3
    frac = excluded / max(1, total)
    print(f"router near-ties excluded: {excluded}/{total} = {frac:.4f}")
    assert frac < 0.10
    return frac


@pytest.mark.gpu
@pytest.mark.slow
def test_full_b1_layer_pins(dg):
    """full_b1: 30 layers over an 8192-token cache, layers 0, 14, 29 against the oracle."""
    W, w, h = _setup(dg, "full_b1")
    try:
        _layer_pins(dg, W, w, h, [0], 0, check=[0])
    finally:
        _release(h, w)


@pytest.mark.gpu
@pytest.mark.slow
def test_full_b16_layer_pins_before_and_after_hand_off(dg):
    """full_b16: 4096 canvas tokens per step (the grouped GEMMs at 32768 expert
    rows), two requests checked per layer, at cache 4096 and after one block's
    hand-off at 4352."""
    W, w, h = _setup(dg, "full_b16")
    S, n, P0, B = W["sampler"], W["model"]["canvas"], W["prompt_len"], W["batch"]
    req = list(range(B))
    try:
        _layer_pins(dg, W, w, h, req, 0, check=[0, 9])
        a = dg.block_args(req, S["max_steps"], S["schedule_steps"], temperature=S["temperature"],
                          logit_scale_growth=S["logit_scale_growth"], stop_threshold=S["stop_threshold"],
                          seed=S["seed"], block=0)
        out = torch.zeros((B, n), dtype=torch.int32, device="cuda")
        dg.dg_generate_block(h, a, out)
        assert all(dg.dg_get_length(h, r) == P0 + n for r in req)
        _layer_pins(dg, W, w, h, req, 1, check=[5, 15])
    finally:
        _release(h, w)


@pytest.mark.gpu
@pytest.mark.slow
def test_full_b1_step_and_block(dg):
    W, w, h = _setup(dg, "full_b1")
    S, n, P0 = W["sampler"], W["model"]["canvas"], W["prompt_len"]
    try:
        for t in (1, 12):
            _check_step(dg, W, w, h, [0], t, 0, S["temperature"], S["logit_scale_growth"] ** (t - 1),
                        O.linear_keep_count(n, t, S["schedule_steps"]), S["stop_threshold"])
        # whole blocks, as the bench runs them: deterministic; the hand-off appends N positions
        a = dg.block_args([0], S["max_steps"], S["schedule_steps"], temperature=S["temperature"],
                          logit_scale_growth=S["logit_scale_growth"], stop_threshold=S["stop_threshold"],
                          seed=S["seed"], block=0)
        outs = []
        for _ in range(2):
            dg.dg_set_length(h, 0, P0)
            out = torch.zeros((1, n), dtype=torch.int32, device="cuda")
            steps = dg.dg_generate_block(h, a, out)
            assert 1 <= steps <= S["max_steps"]
            assert dg.dg_get_length(h, 0) == P0 + n
            outs.append((steps, to_np(out)))
        assert outs[0][0] == outs[1][0] and np.array_equal(outs[0][1], outs[1][1])
        assert outs[0][1].min() >= 0 and outs[0][1].max() < W["model"]["vocab"]
    finally:
        _release(h, w)


@pytest.mark.gpu
@pytest.mark.slow
def test_full_b16_batched_blocks(dg):
    W, w, h = _setup(dg, "full_b16")
    S, n, P0, B = W["sampler"], W["model"]["canvas"], W["prompt_len"], W["batch"]
    req = list(range(B))
    try:
        # one batched step of block 0, checked on sampled positions of three requests
        got = _check_step(dg, W, w, h, req, 1, 0, S["temperature"], 1.0,
                          O.linear_keep_count(n, 1, S["schedule_steps"]), S["stop_threshold"], check=[0, 7, 15])
        assert got["stop"].sum() == 0                      # stop disabled
        # the four blocks: 12 fixed steps each, every request advances by N per hand-off
        first = None
        for blk in range(W["blocks"]):
            a = dg.block_args(req, S["max_steps"], S["schedule_steps"], temperature=S["temperature"],
                              logit_scale_growth=S["logit_scale_growth"], stop_threshold=S["stop_threshold"],
                              seed=S["seed"], block=blk)
            out = torch.zeros((B, n), dtype=torch.int32, device="cuda")
            assert dg.dg_generate_block(h, a, out) == S["max_steps"]
            for r in req:
                assert dg.dg_get_length(h, r) == P0 + (blk + 1) * n
            if blk == 0:
                first = to_np(out)
        # block 0 again from the same cache state gives the same tokens
        for r in req:
            dg.dg_set_length(h, r, P0)
        a = dg.block_args(req, S["max_steps"], S["schedule_steps"], temperature=S["temperature"],
                          logit_scale_growth=S["logit_scale_growth"], stop_threshold=S["stop_threshold"],
                          seed=S["seed"], block=0)
        out = torch.zeros((B, n), dtype=torch.int32, device="cuda")
        dg.dg_generate_block(h, a, out)
        assert np.array_equal(to_np(out), first)
    finally:
        _release(h, w)
