"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of an oracle function, on the CPU, and
runs the pins that guard it: at least one must fail.  A mistake no pin
catches would be a function whose parity rests on nothing.  The mistakes are
the kind a restatement of the method could make: a dropped term, a wrong sign,
index or shift, a transposed operand, a tie broken the wrong way, a block
scale applied along the wrong axis.  (The planted versions live only in this
file and only while a case runs.)
"""
import math

import numpy as np
import pytest

from oracle import dg_oracle as O
from oracle import nvfp4 as N
from tests import test_oracle_nvfp4 as PN
from tests import test_oracle_pins as P

# the unaltered functions, for planted versions that wrap them
_philox, _router, _attention = O.philox4x32_10, O.router, O.attention
_position_stats, _anneal = O.position_stats, O.anneal_temperature
_quantize = N.quantize
_expert_order = O.expert_order


def _rope_sign(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    theta = base ** (-2.0 * np.arange(half) / x.shape[-1])
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)         # rotation the wrong way


def _rope_interleaved(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    theta = base ** (-2.0 * np.arange(hd // 2) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., 0::2], x[..., 1::2]                                         # pairs (0,1), (2,3), ...
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = x1 * c - x2 * s, x2 * c + x1 * s
    return out


def _attention_scale(q, k, v, allowed=None):
    return _attention(q * math.sqrt(q.shape[-1]) / q.shape[-1], k, v, allowed)   # 1/hd, not 1/sqrt(hd)


def _attention_interleaved_gqa(q, k, v, allowed=None):
    hq, hkv = q.shape[0], k.shape[0]
    heads = [_attention(q[h:h + 1], k[h % hkv:h % hkv + 1], v[h % hkv:h % hkv + 1], allowed)
             for h in range(hq)]                                                 # head h -> KV head h mod Hkv
    return np.concatenate(heads, axis=0)


def _router_softmax_all(x, w, b, k):
    ids, _, g, margin = _router(x, w, b, k)
    p = np.exp(g - g.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return ids, np.take_along_axis(p, ids, axis=1), g, margin                   # softmax over all experts


def _router_high_ties(x, w, b, k):
    g = x @ w.T + (0 if b is None else b)
    idx = np.arange(g.shape[1])
    ids = np.stack([np.lexsort((-idx, -row))[:k] for row in g])                  # ties -> higher id
    sel = np.take_along_axis(g, ids, axis=1)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    return ids, e / e.sum(axis=1, keepdims=True), g, np.full(g.shape[0], np.inf)


def _select_high_ties(g, k):
    g = np.asarray(g, np.float64)
    idx = np.arange(g.shape[1])
    ids = np.stack([np.lexsort((-idx, -row))[:k] for row in g])                  # ties -> higher id
    sel = np.take_along_axis(g, ids, axis=1)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    return ids, e / e.sum(axis=1, keepdims=True), np.full(g.shape[0], np.inf)


def _moe_unweighted(x, layer, top_k):
    ids, _, _, _ = O.router(x, layer["router_w"], layer.get("router_b"), top_k)
    out = np.zeros_like(x, dtype=np.float64)
    for e in np.unique(ids):
        tok, _ = np.nonzero(ids == e)
        out[tok] += O.swiglu_expert(x[tok], layer["w_gate"][e], layer["w_up"][e], layer["w_down"][e])
    return out                                                                   # routing weights dropped


def _swiglu_swapped(x, w_gate, w_up, w_down):
    return ((x @ w_gate.T) * O.silu(x @ w_up.T)) @ w_down.T                       # silu on the wrong branch


def _stats_no_log_s(row, temperature, scale):
    st = dict(_position_stats(row, temperature, scale))
    if st["e"] is not None:
        st["H"] = st["H"] - math.log(st["S"])                                    # the log S term dropped
    return st


def _stats_times_t(row, temperature, scale):
    return _position_stats(row, 1.0 / temperature if temperature else 0.0, scale)   # z = l * T


def _icdf_exclusive(e, S, u):
    c = np.cumsum(e) - e                                                         # exclusive prefix
    j = int(np.searchsorted(c, u * S, side="right"))
    return min(j, len(e) - 1), 0.0


def _keep_high_ties(pmax, k):
    n = len(pmax)
    order = np.lexsort((-np.arange(n), -np.asarray(pmax)))                        # ties -> higher index
    keep = np.zeros(n, dtype=bool)
    keep[order[:k]] = True
    return keep, math.inf


def _budget_exclusive(ent, budget):
    ent = np.asarray(ent, dtype=np.float64)
    order = np.lexsort((np.arange(len(ent)), ent))
    keep = np.zeros(len(ent), dtype=bool)
    run = 0.0
    for i in order:
        if run > budget:                                                         # the position's own H left out
            break
        run += ent[i]
        keep[i] = True
    return keep, math.inf


def _budget_may_keep_none(ent, budget):
    ent = np.asarray(ent, dtype=np.float64)
    order = np.lexsort((np.arange(len(ent)), ent))
    keep = np.zeros(len(ent), dtype=bool)
    run = 0.0
    for i in order:
        if run + ent[i] > budget:                                               # the most certain one not forced
            break
        run += ent[i]
        keep[i] = True
    return keep, math.inf


def _argmax_last_tie(logits):
    z = np.asarray(logits)
    return (z.shape[-1] - 1 - np.argmax(z[..., ::-1], axis=-1)).astype(np.int64)  # ties -> higher index


def _quantize_no_448(w):
    q = _quantize(w)
    amax = float(np.max(np.abs(w)))
    return dict(q, g=float(np.float32(amax / 6.0)))                               # per-tensor scale without E4M3's range


def _ar_no_append(self, req, token):
    return self.denoise_forward(req, [int(token)])[0]                            # the token is never cached


def _embed_sc_transposed(self, tokens, prev_pred=None):
    E = self.weights["embed"]
    h = E[np.asarray(tokens)].astype(np.float64)
    if prev_pred is not None:
        h = h + E[np.asarray(prev_pred)] @ self.weights["w_sc"]                  # W_sc not transposed
    return h


def _e4m3_bias8(codes):
    c = np.asarray(codes).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -7), np.ldexp(1.0 + m / 8.0, e - 8))
    mag = np.where((e == 0xF) & (m == 0x7), np.nan, mag)
    return np.where(c & 0x80, -1.0, 1.0) * mag


def _e2m1_ties_up(x):
    x = np.asarray(x, dtype=np.float64)
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = np.minimum(np.abs(x), 6.0)
    d = np.abs(vals[None, :] - a.reshape(-1, 1))
    pick = 7 - np.argmin(d[:, ::-1], axis=1)                                     # ties -> the larger magnitude
    return (pick.reshape(x.shape) | np.where(np.signbit(x), 8, 0)).astype(np.uint8)


def _dequant_tiled(q):
    s = np.tile(N.e4m3_decode(q["scales"]), (1, N.BLOCK))                        # scales along the wrong axis
    return N.e2m1_decode(q["codes"]) * s * q["g"]


def _pack_swapped(codes):
    c = np.asarray(codes).astype(np.uint8)
    return (c[..., 1::2] & 0xF) | ((c[..., 0::2] & 0xF) << 4)


def _expert_order_tokens_descending(ids, n_experts, tile):
    cnt, off, perm, work, touched = _expert_order(ids, n_experts, tile)
    for e in range(n_experts):
        perm[off[e]:off[e + 1]] = perm[off[e]:off[e + 1]][::-1].copy()      # tokens in the wrong order
    return cnt, off, perm, work, touched


def _expert_order_tile_overrun(ids, n_experts, tile):
    cnt, off, perm, work, touched = _expert_order(ids, n_experts, tile)
    return cnt, off, perm, [(e, p0, min(tile, rows + 1)) for e, p0, rows in work], touched   # off by one


KAT = P._kat_rows()

CASES = {
    "philox word order": (O, "philox4x32_10", lambda c, k: _philox(c, k)[..., [1, 0, 2, 3]],
                          [lambda: [P.test_philox_known_answers(*r) for r in KAT]]),
    "uniform u shift": (O, "unit_uniform",
                        lambda w0: (np.asarray(w0, np.uint64) >> np.uint64(9)).astype(np.float64) * 2.0 ** -24,
                        [P.test_uniform_token_is_uniform_chi_square]),
    "re-noise modulo": (O, "uniform_token", lambda w1, v: (np.asarray(w1, np.uint64) % np.uint64(v)).astype(np.int64),
                        [P.test_uniform_token_exact_edges]),
    "rmsnorm without eps": (O, "rms_norm",
                            lambda x, w, eps: np.asarray(x) / np.sqrt(np.mean(np.asarray(x) ** 2, -1, keepdims=True))
                            * w, [P.test_rms_norm_matches_torch]),
    "rope sign": (O, "rope", _rope_sign, [P.test_rope_closed_form_pairs_and_frequencies]),
    "rope pairing": (O, "rope", _rope_interleaved, [P.test_rope_closed_form_pairs_and_frequencies]),
    "attention scale": (O, "attention", _attention_scale, [lambda: P.test_attention_matches_torch_sdpa_gqa(False)]),
    "gqa head map": (O, "attention", _attention_interleaved_gqa, [P.test_gqa_equals_mha_with_duplicated_kv_heads]),
    "router softmax over all": (O, "router", _router_softmax_all,
                                [P.test_router_ties_go_to_lower_id_and_weights_sum_to_one]),
    "router ties": (O, "router", _router_high_ties, [P.test_router_ties_go_to_lower_id_and_weights_sum_to_one]),
    "select ties": (O, "router_select", _select_high_ties,
                    [P.test_router_select_brute_force_with_ties_and_minus_infinity,
                     P.test_router_ties_go_to_lower_id_and_weights_sum_to_one]),
    "expert order tokens descending": (O, "expert_order", _expert_order_tokens_descending,
                                       [lambda: P.test_expert_order_brute_force(1, 40, 3, 9, 4)]),
    "expert tile overrun": (O, "expert_order", _expert_order_tile_overrun,
                            [lambda: P.test_expert_order_brute_force(1, 40, 3, 9, 4)]),
    "moe weights dropped": (O, "moe", _moe_unweighted, [P.test_moe_with_all_experts_is_the_dense_softmax_mixture]),
    "swiglu branch": (O, "swiglu_expert", _swiglu_swapped, [P.test_moe_single_expert_is_a_swiglu_mlp]),
    "entropy without log S": (O, "position_stats", _stats_no_log_s, [P.test_uniform_logits_give_log_v_entropy]),
    "temperature multiplies": (O, "position_stats", _stats_times_t, [lambda: P.test_stats_match_scipy(0.8, 1.0)]),
    "inverse CDF exclusive": (O, "inverse_cdf", _icdf_exclusive, [P.test_inverse_cdf_brute_force_tiny_vocab]),
    "keep ties": (O, "keep_set", _keep_high_ties, [P.test_keep_set_selects_top_confidence_with_lower_index_ties]),
    "keep schedule floor": (O, "linear_keep_count", lambda n, t, tt: min(n, n * t // tt), [P.test_linear_keep_schedule]),
    "budget exclusive": (O, "keep_entropy_budget", _budget_exclusive, [P.test_entropy_budget_keep_worked_example]),
    "anneal reversed": (O, "anneal_temperature", lambda t, tt, a=0.8, b=0.4: _anneal(t, tt, b, a),
                        [P.test_anneal_is_linear_from_08_to_04]),
    "stop ignores argmax": (O, "stop_two_rounds",
                            lambda hp, h, ap, a, tau=0.005: hp is not None and hp < tau and h < tau,
                            [P.test_two_round_stop_truth_table]),
    "self-conditioning transposed": (O.OracleModel, "embed_tokens", _embed_sc_transposed,
                                     [P.test_self_conditioning_term]),
    "e4m3 bias": (N, "e4m3_decode", _e4m3_bias8, [PN.test_e4m3_decode_matches_torch_float8_e4m3fn]),
    "e2m1 ties up": (N, "e2m1_encode", _e2m1_ties_up, [PN.test_e2m1_encode_is_nearest_with_ties_to_even_by_brute_force]),
    "block scale axis": (N, "dequantize", _dequant_tiled, [lambda: PN.test_quantize_reproduces_weights_built_from_codes(0)]),
    "nibble order": (N, "pack", _pack_swapped, [PN.test_pack_nibble_order_and_round_trip]),
    "budget keeps none": (O, "keep_entropy_budget", _budget_may_keep_none,
                          [lambda: P.test_entropy_budget_keep_invariants(0)]),
    "argmax ties": (O, "argmax_tokens", _argmax_last_tie, [P.test_argmax_tokens_takes_the_lower_index_on_ties,
                                                         P.test_sampler_reports_the_argmax_of_z]),
    "AR step not cached": (O.OracleModel, "ar_next_logits", _ar_no_append,
                           [P.test_ar_decode_one_token_at_a_time_equals_one_causal_pass]),
    "global scale range": (N, "quantize", _quantize_no_448,
                           [lambda: PN.test_quantize_reproduces_weights_built_from_codes(0),
                            PN.test_quantize_error_bound_and_structure]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_a_planted_mistake_fails_a_pin(name, monkeypatch):
    target, attr, wrong, pins = CASES[name]
    monkeypatch.setattr(target, attr, wrong)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake '{name}'"


def test_the_pins_pass_on_the_unaltered_oracle():
    for _, _, _, pins in CASES.values():
        for pin in pins:
            pin()
