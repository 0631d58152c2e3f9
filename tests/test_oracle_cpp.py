"""Pins of the C++ oracle (oracle/dg_oracle.cpp), CPU only.

The C++ oracle restates the numpy oracle's definitions in plain float64 loops
(and can evaluate the layer in float32).  It is pinned here against things
other than itself: the published Philox vectors, closed forms (uniform
logits, one-hot logits, T = 0), brute force, and the numpy oracle, which is
itself pinned by tests/test_oracle_pins.py.  Agreement with the numpy oracle
is within float64 rounding (1e-12 max-abs-rel): the two sum in different
orders (numpy's pairwise sums and BLAS products against plain loops), so
bit-equality is not expected; decisions (expert ids, sampled tokens, the keep
set) are compared exactly wherever the numpy oracle's decision margin is above
that rounding.
"""
import math
import os

import numpy as np
import pytest

from discrete_text_diffusion_b200 import synth
from oracle import cpp as K
from oracle import dg_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = synth.WORKLOADS["tiny_fp32"]["model"]


def _kat_rows():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            lhs, rhs = line.split("->")
            a = [int(x, 16) for x in lhs.split()]
            rows.append((a[:4], a[4:], [int(x, 16) for x in rhs.split()]))
    return rows


@pytest.mark.parametrize("ctr,key,want", _kat_rows())
def test_philox_known_answers(ctr, key, want):
    assert [int(x) for x in K.philox(ctr, key)] == want


def test_philox_and_canvas_match_the_numpy_oracle():
    rng = np.random.default_rng(3)
    for _ in range(64):
        ctr = rng.integers(0, 2 ** 32, 4, dtype=np.uint64)
        key = rng.integers(0, 2 ** 32, 2, dtype=np.uint64)
        assert np.array_equal(K.philox(ctr, key), O.philox4x32_10(ctr, key))
    for seed, block, req in [(0, 0, 0), (2 ** 40 + 7, 3, 5)]:
        assert np.array_equal(K.init_canvas(seed, 300, 262144, block, req),
                              O.init_canvas(seed, 300, 262144, block, req))


def test_router_select_against_brute_force_and_numpy():
    rng = np.random.default_rng(5)
    g = rng.standard_normal((64, 16))
    g[3, [2, 9, 11]] = 5.0                      # ties at the top: lower ids first
    g[4, :] = -np.inf
    g[4, [1, 7]] = 0.5                          # fewer finite logits than k
    ids, w = K.router_select(g, 4)
    ids_o, w_o, _ = O.router_select(g, 4)
    assert np.array_equal(ids, ids_o)
    assert np.allclose(w[np.isfinite(w)], w_o[np.isfinite(w_o)], rtol=1e-14, atol=0)
    # brute force on one row: the k largest by (value desc, id asc)
    row = g[0]
    want = sorted(range(16), key=lambda e: (-row[e], e))[:4]
    assert list(ids[0]) == want
    assert math.isclose(w[0].sum(), 1.0, rel_tol=1e-14)
    assert list(ids[3][:3]) == [2, 9, 11]


def _tiny(seed):
    w = synth.to_numpy_weights(synth.make_weights(TINY, seed=seed, dtype="fp32", router_bias=True))
    return w


def _cache(seed, P):
    k, v = synth.normal_kv(TINY["n_kv_heads"], P, TINY["head_dim"], seed=seed, dtype="fp32")
    return k.numpy().astype(np.float64), v.numpy().astype(np.float64)


@pytest.mark.parametrize("causal", [False, True])
def test_layer_matches_the_numpy_oracle(causal):
    w = _tiny(11)
    om = O.OracleModel(dict(TINY), w)
    P, n = 40, 32
    kc, vc = _cache(12, P)
    om.set_kv(0, 0, kc, vc)
    rng = np.random.default_rng(13)
    h = rng.standard_normal((n, TINY["d_model"])) * 0.02
    pos = P + np.arange(n)
    want, k_o, v_o = om.layer(h, 0, 0, pos, causal=causal)
    got, k_c, v_c = K.layer(TINY, w["layers"][0], h, pos, kc, vc, causal)
    assert O.max_abs_rel(got, want) < 1e-12
    assert O.max_abs_rel(k_c, k_o) < 1e-12 and O.max_abs_rel(v_c, v_o) < 1e-12
    # the layer's own contribution (out - in) is what the check must see
    assert O.max_abs_rel(got - h, want - h) < 1e-11
    # float32 evaluation of the same definitions: close, and visibly not float64
    got32, _, _ = K.layer(TINY, w["layers"][0], h, pos, kc, vc, causal, fp32=True)
    err32 = O.max_abs_rel(got32 - h, want - h)
    assert 1e-9 < err32 < 1e-4


def test_layer_with_an_empty_cache_is_pure_self_attention():
    # P = 0 and causal: row 0 sees only itself, so its attention output is its own V
    w = _tiny(21)
    om = O.OracleModel(dict(TINY), w)
    n = 9
    e = np.zeros((TINY["n_kv_heads"], 0, TINY["head_dim"]))
    om.set_kv(0, 0, e, e)
    rng = np.random.default_rng(22)
    h = rng.standard_normal((n, TINY["d_model"])) * 0.05
    want, _, _ = om.layer(h, 0, 0, np.arange(n), causal=True)
    got, _, _ = K.layer(TINY, w["layers"][0], h, np.arange(n), e, e, True)
    assert O.max_abs_rel(got, want) < 1e-12


def test_denoise_forward_matches_the_numpy_oracle():
    w = _tiny(31)
    om = O.OracleModel(dict(TINY), w)
    prompt = synth.uniform_tokens(24, TINY["vocab"], seed=32).numpy()
    om.encode_causal(0, prompt)
    canvas = synth.uniform_tokens(TINY["canvas"], TINY["vocab"], seed=33).numpy()
    prev = synth.uniform_tokens(TINY["canvas"], TINY["vocab"], seed=34).numpy()
    want = om.denoise_forward(0, canvas, prev)
    caches = [(om.k_cache[0][l], om.v_cache[0][l]) for l in range(TINY["n_layers"])]
    got = K.denoise_forward(TINY, w, caches, canvas, prev)
    assert O.max_abs_rel(got, want) < 1e-12


def _logits(n, V, seed):
    lg, _, _ = synth.peaked_logits(1, n, V, seed=seed, peak_max=12.0)
    return lg[0].numpy().astype(np.float64)


@pytest.mark.parametrize("temperature,keep_k", [(1.0, 9), (0.8, 0), (0.8, 37)])
def test_sampler_matches_the_numpy_oracle(temperature, keep_k):
    lg = _logits(37, 5001, 41)
    kw = dict(seed=77, step=3, block=2, req=1, temperature=temperature, logit_scale=1.5, keep_k=keep_k,
              stop_threshold=0.5)
    got = K.sample_canvas(lg, **kw)
    want = O.sample_canvas(lg, **kw)
    assert np.allclose(got["pmax"], want["pmax"], rtol=1e-12, atol=0)
    assert np.allclose(got["H"], want["H"], rtol=1e-12, atol=1e-15)
    sure = want["sample_margin"] > 1e-12
    assert sure.mean() > 0.9
    assert np.array_equal(got["x_hat"][sure], want["x_hat"][sure])
    assert np.array_equal(got["argmax"], want["argmax"])
    if want["keep_margin"] > 1e-12:
        assert np.array_equal(got["keep"], want["keep"])
        assert np.array_equal(got["x_new"][~got["keep"]], want["x_new"][~want["keep"]])
    assert math.isclose(got["mean_H"], want["mean_H"], rel_tol=1e-12)
    assert got["stop"] == want["stop"]


def test_sampler_closed_forms():
    V = 4096
    # uniform logits: pmax = 1/V, H = log V; the draw is floor(u * V)
    got = K.sample_canvas(np.zeros((5, V)), seed=1, step=1, block=0, req=0, temperature=1.0, logit_scale=1.0,
                          keep_k=5, stop_threshold=-1.0)
    assert np.allclose(got["pmax"], 1.0 / V, rtol=1e-12)
    assert np.allclose(got["H"], math.log(V), rtol=1e-12)
    u = O.unit_uniform(O.sampler_words(1, np.arange(5), 1, 0, 0)[:, 0])
    assert np.array_equal(got["x_hat"], np.floor(u * V).astype(np.int64))
    assert not got["stop"]
    # T = 0 with two tied maxima: pmax = 1/2, H = log 2, the lower index drawn
    lg = np.zeros((2, 64))
    lg[:, [5, 40]] = 3.0
    z = K.sample_canvas(lg, seed=1, step=1, block=0, req=0, temperature=0.0, logit_scale=1.0, keep_k=1,
                        stop_threshold=1.0)
    assert np.allclose(z["pmax"], 0.5) and np.allclose(z["H"], math.log(2))
    assert list(z["x_hat"]) == [5, 5]
    assert z["stop"]                            # mean H = log 2 < 1.0
    # a confident canvas (one-hot logits at scale 50): every pmax ~ 1, H ~ 0
    lg = np.full((4, 32), 0.0)
    lg[np.arange(4), [3, 1, 4, 1]] = 50.0
    c = K.sample_canvas(lg, seed=2, step=1, block=0, req=0, temperature=1.0, logit_scale=1.0, keep_k=4,
                        stop_threshold=0.1)
    assert list(c["x_hat"]) == [3, 1, 4, 1] and c["stop"] and c["keep"].all()


def test_full_width_layer_matches_the_numpy_oracle():
    """One layer at the full-width shape (d 2816, 16/8 heads of 256, 128 experts
    top-8, F 704) over a 512-position cache, 64 canvas rows, router bias N(0, 1):
    the C++ float64 loops against the numpy oracle."""
    W = synth.WORKLOADS["layer_bf16"]
    M = dict(W["model"])
    w = synth.to_numpy_weights(synth.make_weights(M, seed=51, dtype="bf16", router_bias=True))
    om = O.OracleModel(dict(M), w)
    k, v = synth.normal_kv(M["n_kv_heads"], 512, M["head_dim"], seed=52, dtype="bf16")
    kc, vc = k.float().numpy().astype(np.float64), v.float().numpy().astype(np.float64)
    om.set_kv(0, 0, kc, vc)
    n = 64
    h = om.embed_tokens(synth.uniform_tokens(n, M["vocab"], seed=53).numpy())
    pos = 512 + np.arange(n)
    want, _, _ = om.layer(h, 0, 0, pos, causal=False)
    got, _, _ = K.layer(M, w["layers"][0], h, pos, kc, vc, False)
    assert O.max_abs_rel(got - h, want - h) < 1e-11
