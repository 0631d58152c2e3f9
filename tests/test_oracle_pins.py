"""Pins of the CPU oracle against things other than itself.

Each check ties an oracle function to a library routine, a closed form, an
invariant or brute force, chosen so that a plausible mistake (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
CPU only.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch
import torch.nn.functional as F

from oracle import dg_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- Philox

def _kat_rows():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            lhs, rhs = line.split("->")
            a = [int(x, 16) for x in lhs.split()]
            b = [int(x, 16) for x in rhs.split()]
            rows.append((a[:4], a[4:], b))
    return rows


@pytest.mark.parametrize("ctr,key,want", _kat_rows())
def test_philox_known_answers(ctr, key, want):
    got = O.philox4x32_10(np.array(ctr), np.array(key))
    assert [int(x) for x in got] == want


def test_philox_broadcast_matches_scalar():
    ctr = np.array([[i, 7, 3, 1] for i in range(5)])
    batch = O.philox4x32_10(ctr, np.array([11, 12]))
    for i in range(5):
        assert np.array_equal(batch[i], O.philox4x32_10(ctr[i], np.array([11, 12])))


def test_uniform_token_is_uniform_chi_square():
    # 2e5 draws over V = 16: a chi-square test at p > 1e-4 (fixed seed -> deterministic)
    w = O.sampler_words(5, np.arange(200_000), 3, 1, 2)
    tok = O.uniform_token(w[:, 1], 16)
    counts = np.bincount(tok, minlength=16)
    assert tok.min() >= 0 and tok.max() < 16
    assert scipy.stats.chisquare(counts).pvalue > 1e-4
    u = O.unit_uniform(w[:, 0])
    assert u.min() >= 0.0 and u.max() < 1.0
    assert scipy.stats.kstest(u, "uniform").pvalue > 1e-4


def test_uniform_token_exact_edges():
    assert O.uniform_token(0, 262144) == 0
    assert O.uniform_token(0xFFFFFFFF, 262144) == 262143
    assert O.uniform_token(0x80000000, 1000) == 500


# --------------------------------------------------------------- RMSNorm/RoPE

def test_rms_norm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(7, 96)) * 3
    w = rng.normal(size=96)
    ref = F.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(w), eps=1e-6).numpy()
    assert np.allclose(O.rms_norm(x, w, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_rope_position_zero_is_identity_and_norm_preserving():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(3, 5, 64))
    assert np.allclose(O.rope(x, np.zeros(5), 10000.0), x)
    y = O.rope(x, np.array([0, 3, 17, 1000, 8191]), 10000.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1))


def test_rope_closed_form_pairs_and_frequencies():
    # hd = 4: pairs (0,2) with theta_0 = 1 and (1,3) with theta_1 = base^(-1/2) = 0.01.
    e0 = np.array([[1.0, 0, 0, 0]])
    e1 = np.array([[0, 1.0, 0, 0]])
    p = 5.0
    assert np.allclose(O.rope(e0, [p], 10000.0), [[math.cos(p), 0, math.sin(p), 0]])
    assert np.allclose(O.rope(e1, [p], 10000.0), [[0, math.cos(p * 0.01), 0, math.sin(p * 0.01)]])


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(2)
    q = rng.normal(size=(1, 64))
    k = rng.normal(size=(1, 64))
    base = 10000.0
    s0 = (O.rope(q, [40], base) @ O.rope(k, [13], base).T).item()
    for shift in (1, 100, 5000):
        s = (O.rope(q, [40 + shift], base) @ O.rope(k, [13 + shift], base).T).item()
        assert abs(s - s0) < 1e-9


# ------------------------------------------------------------------ attention

def _sdpa(q, k, v, allowed):
    hq, hkv = q.shape[0], k.shape[0]
    kt = torch.from_numpy(k).repeat_interleave(hq // hkv, dim=0)
    vt = torch.from_numpy(v).repeat_interleave(hq // hkv, dim=0)
    mask = None if allowed is None else torch.from_numpy(allowed)
    return F.scaled_dot_product_attention(torch.from_numpy(q), kt, vt, attn_mask=mask).numpy()


@pytest.mark.parametrize("masked", [False, True])
def test_attention_matches_torch_sdpa_gqa(masked):
    rng = np.random.default_rng(3)
    q = rng.normal(size=(8, 11, 32))
    k = rng.normal(size=(2, 19, 32))
    v = rng.normal(size=(2, 19, 32))
    allowed = None
    if masked:
        allowed = np.arange(19)[None, :] <= (8 + np.arange(11))[:, None]
    got = O.attention(q, k, v, allowed)
    assert np.allclose(got, _sdpa(q, k, v, allowed), rtol=1e-10, atol=1e-12)


def test_gqa_equals_mha_with_duplicated_kv_heads():
    rng = np.random.default_rng(4)
    q = rng.normal(size=(4, 6, 16))
    k = rng.normal(size=(2, 9, 16))
    v = rng.normal(size=(2, 9, 16))
    mha = O.attention(q, np.repeat(k, 2, axis=0), np.repeat(v, 2, axis=0))
    assert np.allclose(O.attention(q, k, v), mha)
    # head 1 must read KV head 0 and head 2 KV head 1 (not interleaved)
    assert np.allclose(O.attention(q[1:2], k[0:1], v[0:1]), mha[1:2])
    assert np.allclose(O.attention(q[2:3], k[1:2], v[1:2]), mha[2:3])


def _tiny_model(seed=0, n_layers=1, d=32, hq=4, hkv=2, hd=8, e=4, k=2, f=24, vocab=50, n=6):
    rng = np.random.default_rng(seed)
    cfg = dict(n_layers=n_layers, d_model=d, n_heads=hq, n_kv_heads=hkv, head_dim=hd,
               n_experts=e, top_k=k, d_ff=f, vocab=vocab, canvas=n, rope_base=10000.0,
               rms_eps=1e-6)
    nrm = lambda *s: rng.normal(size=s) * 0.3
    layers = [dict(attn_norm=1 + 0.1 * rng.normal(size=d), wq=nrm(hq * hd, d), wk=nrm(hkv * hd, d),
                   wv=nrm(hkv * hd, d), wo=nrm(d, hq * hd), ffn_norm=1 + 0.1 * rng.normal(size=d),
                   router_w=nrm(e, d), router_b=rng.normal(size=e), w_gate=nrm(e, f, d),
                   w_up=nrm(e, f, d), w_down=nrm(e, d, f)) for _ in range(n_layers)]
    w = dict(embed=rng.normal(size=(vocab, d)), w_sc=nrm(d, d), final_norm=1 + 0.1 * rng.normal(size=d),
             layers=layers)
    return O.OracleModel(cfg, w)


def test_cache_plus_canvas_equals_prefix_lm_attention_over_concatenation():
    """Encoding the prompt causally into the cache and then running the canvas
    bidirectionally over cache + canvas equals ONE pass over [prompt; canvas]
    with a prefix-LM mask (prompt rows causal, canvas rows see everything)."""
    m = _tiny_model(seed=5)
    c = m.cfg
    rng = np.random.default_rng(6)
    prompt = rng.integers(0, c["vocab"], 9)
    canvas = rng.integers(0, c["vocab"], c["canvas"])
    h_prompt = m.encode_causal(0, prompt)
    pos = 9 + np.arange(len(canvas))
    h_canvas, _, _ = m.layer(m.embed_tokens(canvas), 0, 0, pos, causal=False)

    # one pass over the concatenation, written with torch SDPA and an explicit mask
    L = m.weights["layers"][0]
    seq = np.concatenate([prompt, canvas])
    n = len(seq)
    h = m.weights["embed"][seq]
    x = O.rms_norm(h, L["attn_norm"], c["rms_eps"])
    hq, hkv, hd = c["n_heads"], c["n_kv_heads"], c["head_dim"]
    q = O.rope((x @ L["wq"].T).reshape(n, hq, hd).transpose(1, 0, 2), np.arange(n), c["rope_base"])
    k = O.rope((x @ L["wk"].T).reshape(n, hkv, hd).transpose(1, 0, 2), np.arange(n), c["rope_base"])
    v = (x @ L["wv"].T).reshape(n, hkv, hd).transpose(1, 0, 2)
    allowed = np.arange(n)[None, :] <= np.arange(n)[:, None]
    allowed[9:, :] = True
    o = _sdpa(q, k, v, allowed).transpose(1, 0, 2).reshape(n, hq * hd)
    h = h + o @ L["wo"].T
    h = h + O.moe(O.rms_norm(h, L["ffn_norm"], c["rms_eps"]), L, c["top_k"])
    assert np.allclose(h[:9], h_prompt, rtol=1e-10, atol=1e-10)
    assert np.allclose(h[9:], h_canvas, rtol=1e-10, atol=1e-10)


# ------------------------------------------------------------------------ MoE

def test_moe_with_all_experts_is_the_dense_softmax_mixture():
    m = _tiny_model(seed=7, e=4, k=4)
    L = m.weights["layers"][0]
    rng = np.random.default_rng(8)
    x = rng.normal(size=(5, m.cfg["d_model"]))
    g = torch.from_numpy(x @ L["router_w"].T + L["router_b"])
    p = torch.softmax(g, dim=-1)
    xt = torch.from_numpy(x)
    dense = sum(p[:, e:e + 1] * (F.silu(xt @ torch.from_numpy(L["w_gate"][e]).T)
                                 * (xt @ torch.from_numpy(L["w_up"][e]).T))
                @ torch.from_numpy(L["w_down"][e]).T for e in range(4))
    assert np.allclose(O.moe(x, L, 4), dense.numpy(), rtol=1e-10, atol=1e-12)


def test_moe_single_expert_is_a_swiglu_mlp():
    m = _tiny_model(seed=9, e=1, k=1)
    L = m.weights["layers"][0]
    x = np.random.default_rng(10).normal(size=(3, m.cfg["d_model"]))
    xt = torch.from_numpy(x)
    mlp = (F.silu(xt @ torch.from_numpy(L["w_gate"][0]).T) * (xt @ torch.from_numpy(L["w_up"][0]).T)) \
        @ torch.from_numpy(L["w_down"][0]).T
    assert np.allclose(O.moe(x, L, 1), mlp.numpy(), rtol=1e-12, atol=1e-12)


def test_router_ties_go_to_lower_id_and_weights_sum_to_one():
    x = np.eye(1, 3)                    # picks column 0 of w_router^T
    w_router = np.array([[1.0, 0, 0], [2.0, 0, 0], [1.0, 0, 0], [2.0, 0, 0], [0.5, 0, 0]])
    ids, w, g, margin = O.router(x, w_router, None, 3)
    assert ids.tolist() == [[1, 3, 0]]
    assert margin[0] == 0.0             # expert 0 vs 2: an exact tie decided by id
    e = np.exp(np.array([2.0, 2.0, 1.0]) - 2.0)
    assert np.allclose(w[0], e / e.sum()) and abs(w.sum() - 1) < 1e-15


@pytest.mark.parametrize("seed,T,k,E,tile", [(0, 7, 2, 5, 3), (1, 40, 3, 9, 4), (2, 1, 1, 1, 1), (3, 25, 4, 30, 2)])
def test_expert_order_brute_force(seed, T, k, E, tile):
    """The permutation against a sort by (expert, item index) written as a
    plain Python key sort; counts, offsets and work tiles against direct counts."""
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    cnt, off, perm, work, touched = O.expert_order(ids, E, tile)
    items = ids.reshape(-1).tolist()
    want = sorted(range(len(items)), key=lambda i: (items[i], i))
    assert perm.tolist() == want
    assert cnt.tolist() == [items.count(e) for e in range(E)]
    assert off[0] == 0 and all(off[e + 1] - off[e] == cnt[e] for e in range(E)) and off[E] == T * k
    assert touched == len(set(items))
    covered = []
    for e, p0, rows in work:
        assert 1 <= rows <= tile and off[e] <= p0 and p0 + rows <= off[e + 1]
        assert all(items[perm[p]] == e for p in range(p0, p0 + rows))
        covered += list(range(p0, p0 + rows))
    assert covered == list(range(T * k))          # tiles in expert order, no gap, no overlap
    # only each expert's last tile may be short
    for (e, p0, rows), nxt in zip(work, work[1:] + [(None, None, None)]):
        if nxt[0] == e:
            assert rows == tile


def test_router_select_brute_force_with_ties_and_minus_infinity():
    """Selection on given logits against enumeration of every k-subset: the
    chosen set has the largest sum of ranks under (value desc, id asc), listed
    in that order; -inf values rank last, among themselves by id."""
    import itertools
    rng = np.random.default_rng(31)
    for trial in range(40):
        E, k = int(rng.integers(2, 7)), 0
        k = int(rng.integers(1, E + 1))
        g = rng.choice([-np.inf, -1.0, 0.0, 0.5, 2.0], size=(1, E))
        if not np.isfinite(g).any():
            g[0, 0] = 0.0
        ids, w, margin = O.router_select(g, k)
        key = lambda e: (-g[0, e], e)                      # python tuples: -(-inf) = inf sorts last
        ranked = sorted(range(E), key=key)
        best = min(itertools.combinations(range(E), k), key=lambda c: sorted(ranked.index(e) for e in c))
        assert ids[0].tolist() == sorted(best, key=key)
        assert len(set(ids[0].tolist())) == k
        fin = np.isfinite(g[0, ids[0]])
        assert np.all(w[0][~fin] == 0) and abs(w[0].sum() - 1) < 1e-12


def test_moe_is_token_order_invariant():
    m = _tiny_model(seed=11, e=6, k=2)
    L = m.weights["layers"][0]
    x = np.random.default_rng(12).normal(size=(10, m.cfg["d_model"]))
    perm = np.random.default_rng(13).permutation(10)
    assert np.allclose(O.moe(x, L, 2)[perm], O.moe(x[perm], L, 2))


# -------------------------------------------------------------------- sampler

def test_uniform_logits_give_log_v_entropy():
    st = O.position_stats(np.zeros(262144, np.float32), 0.8, 1.0)
    assert abs(st["H"] - math.log(262144)) < 1e-9
    assert abs(st["pmax"] - 1 / 262144) < 1e-15


@pytest.mark.parametrize("temperature,scale", [(1.0, 1.0), (0.8, 1.0), (1.0, 2.25)])
def test_stats_match_scipy(temperature, scale):
    rng = np.random.default_rng(14)
    l = rng.gumbel(size=4096).astype(np.float32)
    st = O.position_stats(l, temperature, scale)
    z = l.astype(np.float64) * scale / temperature
    p = scipy.special.softmax(z)
    assert abs(st["H"] - scipy.stats.entropy(p)) < 1e-10
    assert abs(st["pmax"] - p.max()) < 1e-15


def test_small_temperature_sample_is_argmax():
    rng = np.random.default_rng(15)
    logits = rng.normal(size=(16, 300)).astype(np.float32)
    out = O.sample_canvas(logits, seed=1, step=1, block=0, req=0, temperature=1e-6,
                          logit_scale=1.0, keep_k=4, stop_threshold=-1)
    assert np.array_equal(out["x_hat"], logits.argmax(axis=1))
    out0 = O.sample_canvas(logits, seed=1, step=1, block=0, req=0, temperature=0.0,
                           logit_scale=1.0, keep_k=4, stop_threshold=-1)
    assert np.array_equal(out0["x_hat"], logits.argmax(axis=1))
    assert np.allclose(out0["H"], 0) and np.allclose(out0["pmax"], 1)


def test_zero_temperature_ties_go_to_lower_index():
    l = np.array([[0.0, 3.0, 1.0, 3.0]], np.float32)
    out = O.sample_canvas(l, seed=0, step=1, block=0, req=0, temperature=0.0, logit_scale=1.0,
                          keep_k=1, stop_threshold=-1)
    assert out["x_hat"][0] == 1
    assert abs(out["pmax"][0] - 0.5) < 1e-15 and abs(out["H"][0] - math.log(2)) < 1e-15


def test_inverse_cdf_brute_force_tiny_vocab():
    rng = np.random.default_rng(16)
    for _ in range(200):
        vocab = int(rng.integers(1, 9))
        e = rng.random(vocab)
        e[rng.random(vocab) < 0.2] = 0.0
        if e.sum() == 0:
            e[0] = 1.0
        u = rng.random()
        j, margin = O.inverse_cdf(e, e.sum(), u)
        # enumerate: the token whose half-open CDF interval [C_{j-1}, C_j) holds u*S
        acc, want = 0.0, None
        for i in range(vocab):
            if acc <= u * e.sum() < acc + e[i]:
                want = i
                break
            acc += e[i]
        assert j == want and margin >= 0.0


def test_sample_frequencies_follow_the_distribution():
    logits = np.log(np.array([[0.5, 0.1, 0.25, 0.15, 0.0001]], np.float32))
    p = scipy.special.softmax(logits[0].astype(np.float64))
    n = 50_000
    w = O.sampler_words(77, np.arange(n), 1, 0, 0)
    u = O.unit_uniform(w[:, 0])
    st = O.position_stats(logits[0], 1.0, 1.0)
    draws = np.array([O.inverse_cdf(st["e"], st["S"], ui)[0] for ui in u])
    counts = np.bincount(draws, minlength=5)
    assert scipy.stats.chisquare(counts, p * n).pvalue > 1e-4


def test_keep_set_selects_top_confidence_with_lower_index_ties():
    pmax = np.array([0.2, 0.9, 0.5, 0.9, 0.1, 0.5])
    keep, margin = O.keep_set(pmax, 3)
    assert keep.tolist() == [False, True, True, True, False, False]
    assert margin == 0.0
    keep4, _ = O.keep_set(pmax, 4)
    assert keep4.tolist() == [False, True, True, True, False, True]


def test_keep_set_brute_force_small():
    rng = np.random.default_rng(17)
    for _ in range(100):
        n = int(rng.integers(1, 7))
        k = int(rng.integers(0, n + 1))
        pmax = rng.integers(0, 4, n) / 4.0            # many ties
        keep, _ = O.keep_set(pmax, k)
        assert keep.sum() == k
        # every kept position beats every dropped one by (pmax desc, index asc)
        for i in np.nonzero(keep)[0]:
            for j in np.nonzero(~keep)[0]:
                assert pmax[i] > pmax[j] or (pmax[i] == pmax[j] and i < j)


def test_linear_keep_schedule():
    assert [O.linear_keep_count(32, t, 4) for t in range(1, 5)] == [8, 16, 24, 32]
    assert O.linear_keep_count(256, 48, 48) == 256
    assert O.linear_keep_count(256, 1, 48) == 6


def test_renoise_and_kept_tokens():
    rng = np.random.default_rng(18)
    logits = rng.normal(size=(8, 40)).astype(np.float32)
    out = O.sample_canvas(logits, seed=3, step=2, block=1, req=4, temperature=1.0,
                          logit_scale=1.0, keep_k=3, stop_threshold=0.5)
    w = O.sampler_words(3, np.arange(8), 2, 1, 4)
    assert np.array_equal(out["x_new"][~out["keep"]], O.uniform_token(w[:, 1], 40)[~out["keep"]])
    assert np.array_equal(out["x_new"][out["keep"]], out["x_hat"][out["keep"]])
    assert out["stop"] == (out["H"].mean() < 0.5)


# ------------------------------------------------------------ block behaviour

def test_fully_confident_canvas_stops_at_step_one():
    m = _tiny_model(seed=19, n_layers=2)
    m.encode_causal(0, np.arange(5))
    toks, steps, trace = m.generate_block(0, seed=0, block=0, max_steps=48, schedule_steps=48,
                                          temperature=1.0, logit_scale_growth=1.0,
                                          stop_threshold=0.1, append=False)
    assert steps > 1  # ordinary logits: not confident at step 1
    m2 = _tiny_model(seed=19, n_layers=2)
    m2.weights["embed"] = m2.weights["embed"] * 50.0     # huge logit peaks -> H ~ 0
    m2.encode_causal(0, np.arange(5))
    toks, steps, trace = m2.generate_block(0, seed=0, block=0, max_steps=48, schedule_steps=48,
                                           temperature=1.0, stop_threshold=0.1, append=False)
    assert steps == 1 and trace[0]["mean_H"] < 1e-6
    assert np.array_equal(toks, trace[0]["x_hat"])


def test_block_appends_causal_encoding_of_its_output():
    m = _tiny_model(seed=20, n_layers=2)
    prompt = np.arange(7) % m.cfg["vocab"]
    m.encode_causal(0, prompt)
    toks, steps, trace = m.generate_block(0, seed=4, block=0, max_steps=3, schedule_steps=3,
                                          temperature=1.0, stop_threshold=-1.0)
    assert steps == 3 and m.length(0) == 7 + m.cfg["canvas"]
    assert np.array_equal(toks, trace[-1]["x_hat"])
    assert trace[-1]["keep"].all()                       # t = T keeps everything
    ref = _tiny_model(seed=20, n_layers=2)
    ref.encode_causal(0, np.concatenate([prompt, toks]))  # one causal pass over all
    for li in range(2):
        assert np.allclose(ref.k_cache[0][li], m.k_cache[0][li], atol=1e-10)
        assert np.allclose(ref.v_cache[0][li], m.v_cache[0][li], atol=1e-10)
    # the canvas of step t+1 is step t's re-noised x_new; self-cond input is x_hat
    assert np.array_equal(trace[1]["canvas_in"], trace[0]["x_new"])


def test_self_conditioning_term():
    m = _tiny_model(seed=21)
    toks = np.array([1, 2, 3])
    prev = np.array([4, 5, 6])
    E, W = m.weights["embed"], m.weights["w_sc"]
    got = m.embed_tokens(toks, prev)
    want = torch.from_numpy(E[toks]) + F.linear(torch.from_numpy(E[prev]), torch.from_numpy(W))
    assert np.allclose(got, want.numpy())
    assert np.allclose(m.embed_tokens(toks), E[toks])


# ------------------------------------------------ the page's sampler variants

def test_entropy_budget_keep_worked_example():
    # sorted: 0.01 (pos 1), 0.03 (pos 3), 0.05 (pos 0) -> running 0.01, 0.04, 0.09 <= 0.1; +0.2 crosses
    keep, margin = O.keep_entropy_budget([0.05, 0.01, 0.2, 0.03], 0.1)
    assert keep.tolist() == [True, True, False, True]
    assert margin == pytest.approx((0.29 - 0.1) / 0.1)
    # a tie at the boundary goes to the lower index
    keep, _ = O.keep_entropy_budget([0.04, 0.05, 0.05, 0.0], 0.1)
    assert keep.tolist() == [True, True, False, True]


@pytest.mark.parametrize("seed", range(5))
def test_entropy_budget_keep_invariants(seed):
    rng = np.random.default_rng(seed)
    ent = np.round(rng.exponential(0.02, 64), 3)          # rounding makes ties
    for budget in (0.0, 0.05, 0.1, 0.3, 10.0):
        keep, _ = O.keep_entropy_budget(ent, budget)
        kept, rest = np.nonzero(keep)[0], np.nonzero(~keep)[0]
        assert len(kept) >= 1                                   # the most certain position is always locked
        assert len(kept) == 1 or ent[kept].sum() <= budget + 1e-12
        if len(rest):
            # every kept position precedes every rejected one in (entropy, index) order ...
            first = min(rest, key=lambda i: (ent[i], i))
            assert all((ent[i], i) < (ent[first], first) for i in kept)
            # ... and the first rejected one does not fit the budget
            assert ent[kept].sum() + ent[first] > budget
        else:
            assert ent.sum() <= budget
    # a budget nothing fits keeps exactly the most certain position (ties -> lower index)
    keep, _ = O.keep_entropy_budget(ent, -1.0)
    assert np.nonzero(keep)[0].tolist() == [int(np.lexsort((np.arange(len(ent)), ent))[0])]
    assert O.keep_entropy_budget([0.5, 0.2, 0.2, 0.9], 0.0)[0].tolist() == [False, True, False, False]
    assert O.keep_entropy_budget([], 0.1)[0].size == 0


def test_anneal_is_linear_from_08_to_04():
    assert O.anneal_temperature(1, 48) == pytest.approx(0.8)
    assert O.anneal_temperature(48, 48) == pytest.approx(0.4)
    mid = O.anneal_temperature(1, 3), O.anneal_temperature(2, 3), O.anneal_temperature(3, 3)
    assert mid == pytest.approx((0.8, 0.6, 0.4))
    ts = [O.anneal_temperature(t, 48) for t in range(1, 49)]
    steps = np.diff(ts)
    assert np.allclose(steps, steps[0]) and steps[0] < 0


def test_two_round_stop_truth_table():
    a = np.array([3, 1, 4])
    b = np.array([3, 1, 5])
    assert O.stop_two_rounds(0.001, 0.002, a, a.copy())
    assert not O.stop_two_rounds(0.001, 0.002, a, b)          # argmax changed
    assert not O.stop_two_rounds(0.01, 0.002, a, a.copy())    # previous round too uncertain
    assert not O.stop_two_rounds(0.001, 0.006, a, a.copy())   # this round too uncertain
    assert not O.stop_two_rounds(None, 0.001, None, a)        # first round


def test_argmax_tokens_takes_the_lower_index_on_ties():
    lg = np.array([[0.0, 2.0, 2.0, 1.0], [5.0, 5.0, 5.0, 5.0]])
    assert O.argmax_tokens(lg).tolist() == [1, 0]
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 50))
    assert np.array_equal(O.argmax_tokens(x), torch.from_numpy(x).argmax(-1).numpy())


def test_sampler_with_entropy_budget_keeps_the_budget_set_of_its_own_entropies():
    rng = np.random.default_rng(23)
    logits = rng.standard_normal((12, 40)) * rng.uniform(0.1, 6.0, (12, 1))   # mixed confidence
    kw = dict(seed=3, step=2, block=1, req=0, temperature=0.9, logit_scale=1.0, keep_k=5, stop_threshold=-1.0)
    base = O.sample_canvas(logits, **kw)
    for budget in (0.0, 1.0, 4.0, 1e9):
        out = O.sample_canvas(logits, keep_budget=budget, **kw)
        keep, _ = O.keep_entropy_budget(out["H"], budget)
        assert np.array_equal(out["keep"], keep)
        # keep_k is ignored; the sample, the statistics and the re-noise tokens are the top-k run's
        assert np.array_equal(out["x_hat"], base["x_hat"]) and np.allclose(out["H"], base["H"])
        assert np.array_equal(out["x_new"], np.where(keep, out["x_hat"], base["renoise"]))
    assert O.sample_canvas(logits, keep_budget=1e9, **kw)["keep"].all()
    zero = O.sample_canvas(logits, keep_budget=0.0, **kw)                    # every H > 0 here
    assert np.nonzero(zero["keep"])[0].tolist() == [int(np.argmin(zero["H"]))]


def test_block_with_anneal_runs_each_step_at_the_annealed_temperature():
    def run(**extra):
        m = _tiny_model(seed=24, n_layers=1)
        m.encode_causal(0, np.arange(4))
        # the keep schedule (2 steps) is shorter than the step budget (4): the anneal runs over the budget
        return m.generate_block(0, seed=1, block=0, max_steps=4, schedule_steps=2, temperature=0.8,
                                stop_threshold=-1.0, append=False, **extra)
    toks, steps, trace = run(temperature_end=0.4)
    assert steps == 4
    assert [r["temperature"] for r in trace] == pytest.approx([0.8, 0.8 - 0.4 / 3, 0.8 - 0.8 / 3, 0.4])
    # each step equals a plain step at that temperature from the same canvas and self-conditioning
    m = _tiny_model(seed=24, n_layers=1)
    m.encode_causal(0, np.arange(4))
    prev = None
    for t, r in enumerate(trace, start=1):
        one = m.denoise_step(0, r["canvas_in"], prev, step=t, block=0, seed=1, temperature=r["temperature"],
                             logit_scale=1.0, keep_k=O.linear_keep_count(m.cfg["canvas"], t, 2),
                             stop_threshold=-1.0)
        assert np.array_equal(one["x_new"], r["x_new"]) and np.allclose(one["H"], r["H"])
        prev = r["x_hat"]
    # an anneal whose ends are equal is the constant-temperature block
    a = run(temperature_end=0.8)
    b = run()
    assert a[1] == b[1] and np.array_equal(a[0], b[0])
    # the budget keep plugs into the block: a budget of 0 locks one position a step
    toks, steps, trace = run(keep_budget=0.0)
    assert all(r["keep"].sum() == 1 for r in trace) and np.array_equal(toks, trace[-1]["x_hat"])


def test_sampler_reports_the_argmax_of_z():
    rng = np.random.default_rng(25)
    logits = rng.normal(size=(9, 70)).astype(np.float32)
    logits[2, [5, 40]] = 9.0                                   # a tie: the lower index
    for temperature, scale in ((1.0, 1.0), (0.7, 2.0), (0.0, 1.0)):
        out = O.sample_canvas(logits, seed=2, step=1, block=0, req=0, temperature=temperature, logit_scale=scale,
                              keep_k=3, stop_threshold=-1.0)
        assert np.array_equal(out["argmax"], torch.from_numpy(logits).argmax(-1).numpy())
        assert out["argmax"][2] == 5 and out["argmax_margin"][2] == 0.0
        assert (out["argmax_margin"] >= 0).all()
        if temperature == 0.0:
            assert np.array_equal(out["argmax"], out["x_hat"])


def test_block_with_two_round_stop_follows_the_rule_on_its_own_trace():
    def run(tau, scale=50.0, **kw):
        m = _tiny_model(seed=26, n_layers=1)
        m.weights["embed"] = m.weights["embed"] * scale       # confident logits: mean H near 0
        m.encode_causal(0, np.arange(4))
        return m.generate_block(0, seed=2, block=0, max_steps=6, schedule_steps=1, temperature=0.0,
                                stop_threshold=tau, append=False, two_round_stop=True, **kw)
    toks, steps, trace = run(0.1)
    assert not trace[0]["stop"]                                  # no previous round
    for t in range(1, len(trace)):
        want = O.stop_two_rounds(trace[t - 1]["mean_H"], trace[t]["mean_H"], trace[t - 1]["argmax"],
                                 trace[t]["argmax"], tau=0.1)
        assert trace[t]["stop"] == want
    assert all(not r["stop"] for r in trace[:-1])                # the block ends at its first stop
    assert np.array_equal(toks, trace[-1]["x_hat"])
    # T = 0 and every position kept: the canvas becomes the argmax, so a stop means a fixed point
    if trace[-1]["stop"]:
        assert np.array_equal(trace[-1]["argmax"], trace[-2]["argmax"])
    # a negative threshold disables the stop; the one-round test would stop at step 1 here
    assert run(-1.0)[1] == 6
    m = _tiny_model(seed=26, n_layers=1)
    m.weights["embed"] = m.weights["embed"] * 50.0
    m.encode_causal(0, np.arange(4))
    assert m.generate_block(0, seed=2, block=0, max_steps=6, schedule_steps=1, temperature=0.0,
                            stop_threshold=0.1, append=False)[1] == 1


def test_ar_decode_one_token_at_a_time_equals_one_causal_pass():
    m = _tiny_model(seed=27, n_layers=2)
    rng = np.random.default_rng(28)
    prompt = rng.integers(0, m.cfg["vocab"], 7)
    cont = rng.integers(0, m.cfg["vocab"], 5)
    m.encode_causal(0, prompt)
    steps = np.stack([m.ar_next_logits(0, t) for t in cont])
    ref = _tiny_model(seed=27, n_layers=2)
    h = ref.encode_causal(0, np.concatenate([prompt, cont]))      # the whole sequence in one causal pass
    x = O.rms_norm(h[len(prompt):], ref.weights["final_norm"], ref.cfg["rms_eps"])
    want = torch.from_numpy(x) @ torch.from_numpy(ref.weights["embed"]).T
    assert np.allclose(steps, want.numpy(), rtol=1e-10, atol=1e-10)
    assert m.length(0) == len(prompt) + len(cont)
    for li in range(2):
        assert np.allclose(m.k_cache[0][li], ref.k_cache[0][li], atol=1e-12)
        assert np.allclose(m.v_cache[0][li], ref.v_cache[0][li], atol=1e-12)


def test_certain_and_stable_canvas_stops_after_round_two():
    """[P1 六]: when every prediction is certain and no longer changes (the page's structured-output example),
    the block needs two rounds.  With the layers reduced to the identity (zero O, expert down and
    self-conditioning weights) and large embeddings, each position's logits peak at its own token, so at T = 0
    with every position kept the round-1 argmax is the canvas itself and round 2 repeats it."""
    m = _tiny_model(seed=29, n_layers=2, vocab=40)
    m.weights["embed"] = m.weights["embed"] * 20.0
    m.weights["w_sc"] = np.zeros_like(m.weights["w_sc"])
    for L in m.weights["layers"]:
        L["wo"] = np.zeros_like(L["wo"])
        L["w_down"] = np.zeros_like(L["w_down"])
    m.encode_causal(0, np.arange(5))
    canvas0 = O.init_canvas(4, m.cfg["canvas"], m.cfg["vocab"], 0, 0)
    logits = m.denoise_forward(0, canvas0)
    assert np.array_equal(O.argmax_tokens(logits), canvas0)          # the fixed point the pin relies on
    toks, steps, trace = m.generate_block(0, seed=4, block=0, max_steps=8, schedule_steps=1, temperature=0.0,
                                          stop_threshold=0.005, append=False, two_round_stop=True)
    assert steps == 2 and [r["stop"] for r in trace] == [False, True]
    assert trace[0]["mean_H"] == 0.0 and np.array_equal(toks, canvas0)
