"""The router ([P1 二]: 128 experts, 8 per token) through its C-ABI self-test,
against the oracle.

On identical fp32 gate logits both sides must pick the same experts in the same
order (logit descending, ties to the lower id) for every token whose decision
is not a rounding-order tie; the permutation into expert order, the counts,
offsets, work tiles and the distinct-expert count are integer work and must
equal the oracle's on the GPU's own expert ids, bit for bit.  Cases: the canvas
step (256 tokens) and the batch-16 step (4096 tokens), a router bias that
concentrates every token on four hot experts, planted exact ties, rows with
-inf logits, and the scalar and vector top-k forms (E = 8, 200, 128, 256).
"""
import numpy as np
import pytest
import torch

from oracle import dg_oracle as O
from tests._util import to_np

MARGIN = 1e-5   # decisions closer than this (relative to the logit size) may differ by rounding order


def _run(dg, logits, bias, k, tile):
    T, E = logits.shape
    n_work_max = E + (T * k + tile - 1) // tile
    dev = "cuda"
    out = dict(ids=torch.full((T, k), -1, dtype=torch.int32, device=dev),
               wts=torch.full((T, k), float("nan"), device=dev),
               cnt=torch.full((E,), -1, dtype=torch.int32, device=dev),
               off=torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
               perm=torch.full((T * k,), -1, dtype=torch.int32, device=dev),
               work=torch.full((3 * n_work_max,), -1, dtype=torch.int32, device=dev),
               n_work=torch.zeros(1, dtype=torch.int32, device=dev),
               touched=torch.zeros(1, dtype=torch.int32, device=dev))
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="fp32", max_batch=1, max_ctx=64)
    dg.dg_selftest_router(h, logits.cuda(), None if bias is None else bias.cuda(), k, tile, out)
    dg.dg_synchronize(h)
    h.close()
    return {n: to_np(t) for n, t in out.items()}


def _order_margin(g, k):
    """Per token: the smallest gap between consecutive values of its sorted
    top-(k+1) logits (every gap that decides the selection or its order)."""
    s = -np.sort(-g, axis=1)[:, :min(k + 1, g.shape[1])]
    with np.errstate(invalid="ignore"):
        gaps = np.abs(np.diff(s, axis=1))
    gaps = np.where(np.isnan(gaps), 0.0, gaps)          # -inf vs -inf: an exact tie
    scale = np.maximum(1.0, np.abs(np.where(np.isfinite(s), s, 0)).max(1))
    return gaps.min(1) / scale


def _check(dg, logits, bias, k, tile, expect_exact_all=False):
    T, E = logits.shape
    got = _run(dg, logits, bias, k, tile)
    g64 = logits.double().numpy() + (0.0 if bias is None else bias.double().numpy())
    ids, w, _ = O.router_select(g64, k)
    margin = _order_margin(g64, k)
    # no expert twice in a token, every id in range
    assert (got["ids"] >= 0).all() and (got["ids"] < E).all()
    assert all(len(set(r)) == k for r in got["ids"].tolist())
    bad = (got["ids"] != ids).any(1)
    hard = bad & (margin > MARGIN)
    assert not hard.any(), f"{int(hard.sum())} tokens pick other experts above the margin: {np.nonzero(hard)[0][:10]}"
    if expect_exact_all:
        assert not bad.any()
    same = ~bad
    assert np.allclose(got["wts"][same], w[same], rtol=1e-6, atol=1e-7)
    assert np.allclose(got["wts"].sum(1), 1.0, atol=1e-6)
    # the integer stages, on the GPU's own ids: bit-exact
    cnt, off, perm, work, touched = O.expert_order(got["ids"], E, tile)
    assert np.array_equal(got["cnt"], cnt)
    assert np.array_equal(got["off"], off)
    assert np.array_equal(got["perm"], perm)
    nw = int(got["n_work"][0])
    assert nw == len(work)
    assert np.array_equal(got["work"][:3 * nw].reshape(nw, 3), np.array(work, dtype=np.int64).reshape(nw, 3))
    assert int(got["touched"][0]) == touched == len(np.unique(got["ids"]))
    return got, int(bad.sum())


def _logits(T, E, seed, scale=1.06):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((T, E), generator=g) * scale


@pytest.mark.gpu
@pytest.mark.parametrize("T", [256, 4096])
def test_router_matches_oracle_canvas_and_batch16(dg, T):
    """The full-width router at the canvas step (256 tokens, one permutation
    pass) and at batch 16 (4096 tokens, the chunked permutation), bias N(0,1)."""
    E, k = 128, 8
    logits = _logits(T, E, seed=T)
    bias = torch.randn(E, generator=torch.Generator().manual_seed(T + 1))
    _, low = _check(dg, logits, bias, k, tile=128)
    assert low == 0


@pytest.mark.gpu
@pytest.mark.parametrize("T", [256, 4096])
def test_router_hot_experts(dg, T):
    """A bias that puts four experts in every token's top-8: expert runs of T
    rows, cut into 128-row tiles, next to experts with a few rows."""
    E, k = 128, 8
    logits = _logits(T, E, seed=T + 7)
    bias = torch.zeros(E)
    bias[:4] = 8.0
    got, low = _check(dg, logits, bias, k, tile=128)
    assert low == 0
    assert (got["cnt"][:4] == T).all()


@pytest.mark.gpu
def test_router_exact_ties_go_to_the_lower_id(dg):
    """Planted exact ties at the top-8 boundary, inside the top-8 and at the
    top: the lower expert id wins, the same on both sides."""
    T, E, k = 256, 128, 8
    logits = _logits(T, E, seed=11)
    rng = np.random.default_rng(12)
    lg = logits.numpy()
    for t in range(T):
        order = np.lexsort((np.arange(E), -lg[t]))
        r = t % 3
        a, b = (order[7], order[8]) if r == 0 else (order[2], order[5]) if r == 1 else (order[0], order[1])
        lg[t, max(a, b)] = lg[t, min(a, b)]        # equal values, the higher id copies the lower
        if t % 5 == 0:                             # and a run of equal values across the boundary
            for j in rng.choice(E, 4, replace=False):
                lg[t, j] = lg[t, order[7]]
    got, low = _check(dg, torch.from_numpy(lg), None, k, tile=64, expect_exact_all=True)
    assert low == 0


@pytest.mark.gpu
def test_router_rows_with_minus_infinity(dg):
    """Tokens with fewer finite logits than k: the finite ones first (by value),
    then the lowest ids among the -inf ones; no expert is picked twice and the
    -inf picks get weight 0."""
    T, E, k = 64, 128, 8
    lg = _logits(T, E, seed=21).numpy()
    for t in range(T):
        keep = np.random.default_rng(t).choice(E, size=1 + t % 6, replace=False)
        row = np.full(E, -np.inf, np.float32)
        row[keep] = lg[t, keep]
        lg[t] = row
    got, low = _check(dg, torch.from_numpy(lg), None, k, tile=32, expect_exact_all=True)
    n_fin = np.isfinite(lg).sum(1)
    for t in range(T):
        assert (got["wts"][t, n_fin[t]:] == 0).all()


@pytest.mark.gpu
@pytest.mark.parametrize("E,k,T", [(8, 2, 300), (200, 5, 129), (256, 16, 256), (128, 1, 33)])
def test_router_other_shapes(dg, E, k, T):
    """The scalar top-k form (E not 128/256), the 256-expert vector form, k = 1."""
    logits = _logits(T, E, seed=E * 3 + k)
    bias = torch.randn(E, generator=torch.Generator().manual_seed(E))
    _, low = _check(dg, logits, bias, k, tile=32)
    assert low == 0


@pytest.mark.gpu
def test_router_selftest_refuses_bad_shapes(dg):
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="fp32", max_batch=1, max_ctx=64)
    x = torch.zeros((4, 300), device="cuda")
    out = {n: torch.zeros(4096, dtype=torch.int32, device="cuda") for n, _ in dg.DgRouterOut._fields_}
    with pytest.raises(dg.DgError) as e:
        dg.dg_selftest_router(h, x, None, 8, 128, out)          # E > 256
    assert e.value.code == dg.DG_EINVAL
    with pytest.raises(dg.DgError):
        dg.dg_selftest_router(h, x[:, :16], None, 17, 128, out)   # k > 16
    h.close()
