"""Run a few denoising steps of a full-width model for a profiler to capture.

    python -m discrete_text_diffusion_b200.profile_step [--layers 1] [--cache 8192]
        [--batch 1] [--steps 2] [--hot-experts 16 --hot-bias 3] [--nvfp4]

The model has the full-depth workload's layer shape (d 2816, 16/8 heads of
256, 128 experts top-8, F 704, vocabulary 262144) with `--layers` layers, so
that one process holds a few GB: a capture that replays a kernel many times
saves and restores all of it.  The prompt cache is a seeded N(0,1) cache of
`--cache` positions written with dg_set_kv (no prefill launches), so the
library's launches are exactly the steps': per step and layer, in order,
QKV, RoPE scatter, attention (+ split combine), O, add + RMSNorm, router
logits, top-k, permutation, gather, expert gate/up, expert down, combine;
then the LM head with the sampler statistics, the sampler's merge pass and
its keep / re-noise pass.  The tensor-core GEMM launches of a step are, for
each layer, QKV, O, router, gate/up, down (gemm_tc_kernel<false>) and then
the LM head (gemm_tc_kernel<true>); with --nvfp4 the expert GEMMs are
gemm_fp4_kernel.

--hot-experts / --hot-bias add a bias to the router logits of the first
experts, which concentrates the routing the way the deep layers of the
full-depth model concentrate it (10-20 experts touched per layer instead of
~80 for layer 0 on random tokens).  It prints the experts touched per layer.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
if os.path.dirname(HERE) not in sys.path:
    sys.path.insert(0, os.path.dirname(HERE))

import discrete_text_diffusion_b200 as dg  # noqa: E402
from discrete_text_diffusion_b200 import synth  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=1)
    ap.add_argument("--cache", type=int, default=8192)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--hot-experts", type=int, default=0)
    ap.add_argument("--hot-bias", type=float, default=3.0)
    ap.add_argument("--nvfp4", action="store_true")
    args = ap.parse_args(argv)
    M = dict(synth.FULL_SHAPE, n_layers=args.layers)
    n, B = M["canvas"], args.batch
    w = synth.make_weights(M, seed=3, dtype="bf16", router_bias=True, device="cuda")
    for L in w["layers"]:
        L["router_b"][:args.hot_experts] += args.hot_bias
    fmt = dg.DG_EXPERT_DTYPE
    if args.nvfp4:
        for L in w["layers"]:
            for name in ("w_gate", "w_up", "w_down"):
                x = L[name]
                e, rows, K = x.shape
                codes = torch.empty((e, rows, K // 2), dtype=torch.uint8, device="cuda")
                scales = torch.empty(dg.nvfp4_scales_shape(e, rows, K), dtype=torch.uint8, device="cuda")
                g = torch.empty(e, dtype=torch.float32, device="cuda")
                dg.dg_quantize_nvfp4(x, codes, scales, g)
                L[name], L[name + "_sf"], L[name + "_g"] = codes, scales, g
        torch.cuda.synchronize()
        fmt = dg.DG_EXPERT_NVFP4
    max_ctx = (args.cache + n + 63) // 64 * 64
    h = dg.dg_create(M, w, dtype="bf16", max_batch=B, max_ctx=max_ctx, expert_format=fmt)
    for r in range(B):
        for li in range(args.layers):
            k, v = synth.normal_kv(M["n_kv_heads"], args.cache, M["head_dim"], seed=100 + 7 * r + li, dtype="bf16",
                                   device="cuda")
            dg.dg_set_kv(h, r, li, k, v)
        dg.dg_set_length(h, r, args.cache)
    dg.dg_synchronize(h)
    launches0 = dg.dg_launch_count(h)
    canvas = synth.uniform_tokens(n, M["vocab"], seed=5, batch=B, device="cuda")
    touched = torch.zeros(args.layers, dtype=torch.int32, device="cuda")
    for t in range(1, args.steps + 1):
        sp = dg.sampler_params(temperature=1.0, keep_k=n * t // (args.steps + 1), seed=3)
        dg.dg_denoise_step(h, list(range(B)), canvas, None, t, sp, dg.step_out(experts_touched=touched))
    dg.dg_synchronize(h)
    print(json.dumps({"layers": args.layers, "cache": args.cache, "batch": B, "steps": args.steps,
                      "launches_per_step": (dg.dg_launch_count(h) - launches0) // args.steps,
                      "experts_touched": touched.tolist(), "nvfp4": args.nvfp4}))
    h.close()


if __name__ == "__main__":
    main()
