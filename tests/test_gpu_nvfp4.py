"""NVFP4 expert weights ([P2] 推荐的部署与优化方案, [P4] MoE 26B参数架构分析)
through the C ABI.

- dg_quantize_nvfp4 against the oracle's quantiser (oracle/nvfp4.py, pinned to
  the OCP MX / OFP8 definitions), bit for bit: element codes, block scales and
  per-matrix scales, on random weights, a full expert matrix, planted rounding
  ties of both encoders, -0.0, zero blocks and an all-zero matrix.
- The NVFP4 grouped expert GEMMs: the full-width layer with NVFP4 experts
  against the oracle's layer on the dequantised weights (max-abs-rel 2e-2, the
  router-margin rule), with and without hot experts; a small bf16 model's whole
  step against the oracle, and its blocks deterministic.
"""
import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from oracle import dg_oracle as O
from oracle import nvfp4 as N
from tests._util import max_abs_rel, to_np

TOL_BF16 = 2e-2
ROUTER_MARGIN = 0.02


def _quantize_gpu(dg, w):
    """w [n, rows, K] bf16 (device) -> (codes, scales, g) device tensors."""
    n, rows, K = w.shape
    codes = torch.empty((n, rows, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.full(dg.nvfp4_scales_shape(n, rows, K), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty(n, dtype=torch.float32, device="cuda")
    dg.dg_quantize_nvfp4(w, codes, scales, g)
    torch.cuda.synchronize()
    return codes, scales, g


def _untile_scales(scales, rows):
    """[n, K/64, rows_pad, 4] -> [n, rows, K/16] (the oracle's layout)."""
    s = scales.permute(0, 2, 1, 3)
    return s.reshape(s.shape[0], s.shape[1], -1)[:, :rows]


def _check_against_oracle(dg, w):
    codes, scales, g = _quantize_gpu(dg, w.cuda())
    n, rows, K = w.shape
    sc = to_np(_untile_scales(scales, rows))
    pad = to_np(scales.permute(0, 2, 1, 3))[:, rows:]
    assert (pad == 0).all(), "padding rows of the scale tiles must be 0"
    for i in range(n):
        q = N.quantize(w[i].float().numpy())
        assert np.float32(q["g"]) == to_np(g)[i], f"matrix {i}: g {to_np(g)[i]} vs {q['g']}"
        assert np.array_equal(sc[i], q["scales"]), f"matrix {i}: block scales differ"
        assert np.array_equal(to_np(codes[i]), N.pack(q["codes"])), f"matrix {i}: codes differ"


@pytest.mark.gpu
@pytest.mark.parametrize("n,rows,K,std", [(2, 200, 128, 1.0), (3, 5, 64, 0.02), (1, 704, 2816, 0.02)])
def test_quantizer_matches_oracle_random(dg, n, rows, K, std):
    g = torch.Generator().manual_seed(rows * 7 + K)
    w = (torch.randn((n, rows, K), generator=g) * std)
    w[:, :, :16] *= 40.0           # a wide dynamic range across blocks
    _check_against_oracle(dg, w.to(torch.bfloat16))


@pytest.mark.gpu
def test_quantizer_ties_signed_zero_and_zero_blocks(dg):
    """Matrix amax 2.625 gives g = 2^-10 exactly.  Block 1: scale 1.0 and
    elements at every E2M1 rounding tie (0.25 .. 5) x 2^-10, both signs, and
    -0.0.  Block 2: amax at the E4M3 midpoint between 1.0 and 1.125 (ties to
    the even code).  Block 3: all zero.  A second matrix is all zero."""
    K = 64
    w = torch.zeros((2, 2, K), dtype=torch.float32)
    u = 2.0 ** -10
    w[0, 0, 0] = 2.625                                  # matrix amax -> g = 2^-10
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    blk = [6.0 * u] + [t * u for t in ties] + [-t * u for t in ties] + [-0.0]
    w[0, 0, 16:32] = torch.tensor(blk)
    w[0, 1, 0] = 6.0 * u * 1.0625                       # E4M3 tie between 1.0 and 1.125
    w[0, 1, 1:16] = torch.linspace(-0.004, 0.004, 15)
    # w[0, 1, 16:32] stays zero: a zero block
    _check_against_oracle(dg, w.to(torch.bfloat16))


def _nvfp4_layer(dg, L):
    """Quantise one layer's expert stacks on the device; returns the device
    entries for the handle and, for the oracle, accessors of the dequantised
    experts (float64, from the device codes)."""
    out, acc = {}, {}
    for name in ("w_gate", "w_up", "w_down"):
        codes, scales, g = _quantize_gpu(dg, L[name])
        out[name], out[name + "_sf"], out[name + "_g"] = codes, scales, g
        acc[name] = _Dequant(codes, scales, g, L[name].shape[1])
    return out, acc


class _Dequant:
    """Expert e of a quantised stack as the oracle's dequantised matrix."""

    def __init__(self, codes, scales, g, rows):
        self.codes, self.scales, self.g, self.rows = codes, scales, g, rows
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            sc = to_np(_untile_scales(self.scales[e:e + 1], self.rows))[0]
            q = dict(codes=N.unpack(to_np(self.codes[e])), scales=sc, g=float(to_np(self.g)[e]))
            self.cache[e] = N.dequantize(q)
        return self.cache[e]


@pytest.mark.gpu
@pytest.mark.parametrize("hot_experts", [0, 4])
def test_full_width_layer_with_nvfp4_experts(dg, hot_experts):
    W = synth.WORKLOADS["layer_bf16"]
    M = W["model"]
    w = synth.make_weights(M, seed=W["seed"], dtype="bf16", router_bias=True, device="cuda")
    if hot_experts:
        w["layers"][0]["router_b"][:hot_experts] += 8.0
    q, acc = _nvfp4_layer(dg, w["layers"][0])
    L = dict(w["layers"][0])
    L.update(q)
    wq = dict(w)
    wq["layers"] = [L]
    k, v = synth.normal_kv(M["n_kv_heads"], W["cache_len"], M["head_dim"], seed=W["seed"] + 50, dtype="bf16",
                           device="cuda")
    h = dg.dg_create(M, wq, dtype="bf16", max_batch=1, max_ctx=W["cache_len"] + M["canvas"],
                     expert_format=dg.DG_EXPERT_NVFP4)
    dg.dg_set_kv(h, 0, 0, k, v)
    dg.dg_set_length(h, 0, W["cache_len"])
    n, V, d = M["canvas"], M["vocab"], M["d_model"]
    canvas = synth.uniform_tokens(n, V, seed=W["seed"] + 1)
    hid = torch.zeros((n, d), device="cuda")
    ids = torch.zeros((n, M["top_k"]), dtype=torch.int32, device="cuda")
    sp = dg.sampler_params(temperature=1.0, keep_k=64, seed=1)
    dg.dg_denoise_step(h, [0], canvas[None].cuda(), None, 1, sp, dg.step_out(), hidden_out=hid,
                       dump=dg.layer_dump(0, expert_ids=ids))
    dg.dg_synchronize(h)
    h.close()
    lw = {kk: (None if t is None else to_np(t.float())) for kk, t in w["layers"][0].items()
          if kk not in ("w_gate", "w_up", "w_down")}
    lw.update(acc)
    om = O.OracleModel(dict(M), {"layers": [lw], "embed": to_np(w["embed"].float()),
                                 "w_sc": None, "final_norm": to_np(w["final_norm"])})
    om.set_kv(0, 0, to_np(k.float()), to_np(v.float()))
    hx = om.embed_tokens(canvas.numpy())
    tr = {}
    ref, _, _ = om.layer(hx, 0, 0, W["cache_len"] + np.arange(n), causal=False, trace=tr)
    gids = to_np(ids)
    same = np.array([set(a) == set(b) for a, b in zip(gids.tolist(), tr["router_ids"].tolist())])
    assert (tr["router_margin"][~same] < ROUTER_MARGIN).all()
    assert same.mean() > 0.9
    got = to_np(hid).astype(np.float64)
    err = float(np.max(np.abs(got[same] - ref[same])) / np.max(np.abs(ref)))
    assert err < TOL_BF16, f"layer output max-abs-rel {err}"
    dref = ref - hx
    derr = float(np.max(np.abs((got - hx)[same] - dref[same])) / np.max(np.abs(dref)))
    assert derr < TOL_BF16, f"layer delta max-abs-rel {derr}"


@pytest.mark.gpu
def test_small_model_with_nvfp4_experts_step_and_blocks(dg):
    M = dict(n_layers=2, d_model=256, n_heads=2, n_kv_heads=1, head_dim=256, n_experts=16, top_k=4, d_ff=128,
             vocab=4096, canvas=32, rope_base=10000.0, rms_eps=1e-6)
    w = synth.make_weights(M, seed=70, dtype="bf16", router_bias=True, device="cuda")
    wq = dict(w)
    wq["layers"] = []
    accs = []
    for L in w["layers"]:
        q, acc = _nvfp4_layer(dg, L)
        L2 = dict(L)
        L2.update(q)
        wq["layers"].append(L2)
        accs.append(acc)
    h = dg.dg_create(M, wq, dtype="bf16", max_batch=1, max_ctx=256, expert_format=dg.DG_EXPERT_NVFP4)
    prompt = synth.uniform_tokens(40, M["vocab"], seed=71)
    dg.dg_prefill_prompt(h, [0], prompt[None].cuda())
    canvas = synth.uniform_tokens(M["canvas"], M["vocab"], seed=72)
    logits = torch.zeros((1, M["canvas"], M["vocab"]), device="cuda")
    dg.dg_denoise_step(h, [0], canvas[None].cuda(), None, 1, dg.sampler_params(keep_k=8, seed=3),
                       dg.step_out(), logits_out=logits)
    dg.dg_synchronize(h)
    layers = []
    for L, acc in zip(w["layers"], accs):
        lw = {kk: (None if t is None else to_np(t.float())) for kk, t in L.items()
              if kk not in ("w_gate", "w_up", "w_down")}
        lw.update(acc)
        layers.append(lw)
    om = O.OracleModel(dict(M), {"layers": layers, "embed": to_np(w["embed"].float()),
                                 "w_sc": to_np(w["w_sc"].float()), "final_norm": to_np(w["final_norm"])})
    om.encode_causal(0, prompt.numpy())
    ref = om.denoise_forward(0, canvas.numpy())
    err = max_abs_rel(to_np(logits)[0], ref)
    assert err < TOL_BF16, f"logits max-abs-rel {err}"
    # whole blocks through the fused head are deterministic
    a = dg.block_args([0], 8, 8, temperature=1.0, stop_threshold=-1.0, seed=5, block=0)
    outs = []
    for _ in range(2):
        dg.dg_set_length(h, 0, 40)
        out = torch.zeros((1, M["canvas"]), dtype=torch.int32, device="cuda")
        dg.dg_generate_block(h, a, out)
        outs.append(to_np(out))
    assert np.array_equal(outs[0], outs[1])
    h.close()
