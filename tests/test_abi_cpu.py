"""The C ABI library loads, exports every function include/dg.h declares, the
ctypes structures match the header's layout, and host-side validation rejects
bad configurations before touching a GPU.  CPU only."""
import ctypes as C
import os
import re
import subprocess

import pytest

import discrete_text_diffusion_b200 as dgm
from discrete_text_diffusion_b200 import dg as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from discrete_text_diffusion_b200 import build
        build.build()
    return B.lib()


def test_every_declared_function_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)


def test_binding_has_same_names_as_abi():
    for n in B.EXPORTS:
        assert callable(getattr(B, n)), n


_STRUCTS = {
    "dg_config": B.DgConfig, "dg_layer_weights": B.DgLayerWeights, "dg_weights": B.DgWeights,
    "dg_sampler_params": B.DgSamplerParams, "dg_step_out": B.DgStepOut, "dg_step_args": B.DgStepArgs,
    "dg_block_args": B.DgBlockArgs, "dg_profile_entry": B.DgProfileEntry,
    "dg_layer_dump": B.DgLayerDump, "dg_router_out": B.DgRouterOut,
}


def test_struct_layouts_match_header(tmp_path):
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void) {"]
    for cname, py in _STRUCTS.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname}.{fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(line.rsplit(" ", 1) for line in out if line)
    for cname, py in _STRUCTS.items():
        assert int(got[f"{cname} size"]) == C.sizeof(py), cname
        for fname, _ in py._fields_:
            assert int(got[f"{cname}.{fname}"]) == getattr(py, fname).offset, f"{cname}.{fname}"


def _create_rc(**over):
    m = dict(dgm.synth.WORKLOADS["tiny_fp32"]["model"])
    m.update(over)
    cfg = B._cfg(m, dtype="fp32", max_batch=1, max_ctx=128)
    out = C.c_void_p()
    rc = B.lib().dg_create(C.byref(cfg), None, None, C.byref(out))
    return rc, B.lib().dg_last_error(None).decode()


@pytest.mark.parametrize("over,word", [
    (dict(n_kv_heads=3), "shape"),
    (dict(head_dim=7), "shape"),
    (dict(top_k=9), "shape"),
    (dict(canvas=0), "canvas"),
])
def test_create_rejects_bad_shapes_on_host(lib, over, word):
    rc, msg = _create_rc(**over)
    assert rc == B.DG_EINVAL and word in msg


def test_create_rejects_missing_weights_on_host(lib):
    rc, msg = _create_rc()
    assert rc == B.DG_EINVAL and "weight" in msg


def test_create_rejects_bad_dtype_and_capacity(lib):
    m = dgm.synth.WORKLOADS["tiny_fp32"]["model"]
    cfg = B._cfg(m, dtype="fp32", max_batch=1, max_ctx=100)     # not a multiple of 64
    out = C.c_void_p()
    assert lib.dg_create(C.byref(cfg), None, None, C.byref(out)) == B.DG_EINVAL
    cfg = B._cfg(m, dtype="fp32", max_batch=65, max_ctx=128)    # too many request slots
    assert lib.dg_create(C.byref(cfg), None, None, C.byref(out)) == B.DG_EINVAL
    cfg = B._cfg(m, dtype="fp32", max_batch=1, max_ctx=128)
    cfg.dtype = 7
    assert lib.dg_create(C.byref(cfg), None, None, C.byref(out)) == B.DG_EINVAL
    cfg = B._cfg(dict(m, d_model=96), dtype="bf16", max_batch=1, max_ctx=128)
    lw = (B.DgLayerWeights * 2)()
    w = B.DgWeights(16, 16, 16, lw)
    rc = lib.dg_create(C.byref(cfg), C.byref(w), None, C.byref(out))
    assert rc == B.DG_EINVAL and "multiples of 64" in lib.dg_last_error(None).decode()


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.dg_synchronize(None) == B.DG_EINVAL
    assert lib.dg_set_length(None, 0, 0) == B.DG_EINVAL
    assert lib.dg_launch_count(None) == 0
    lib.dg_destroy(None)


def test_profile_classes_follow_header():
    import re
    hdr = open(os.path.join(os.path.dirname(B.LIB_PATH), "..", "include", "dg.h")).read()
    vals = {m.group(1).lower(): int(m.group(2)) for m in re.finditer(r"DG_PROF_(\w+) = (\d+)", hdr)}
    count = vals.pop("count")
    assert count == len(B.PROFILE_CLASSES)
    assert [c for c, _ in sorted(vals.items(), key=lambda x: x[1])] == list(B.PROFILE_CLASSES)


def _noalloc(lib, logits, B, n, V, req, sp, canvas):
    err = C.create_string_buffer(256)
    rc = lib.dg_sample_noalloc(logits, B, n, V, (C.c_int * max(1, len(req)))(*req), 1,
                               C.byref(sp) if sp is not None else None, canvas, None, None, err, 256)
    return rc, err.value.decode()


def test_noalloc_sampler_refuses_bad_arguments_on_host(lib):
    """Every check of dg_sample_noalloc runs before its first CUDA call: these
    refusals need no GPU (the pointers are never dereferenced)."""
    fake = C.c_void_p(0x10000)        # 16-byte aligned, never touched
    sp = B.sampler_params(temperature=1.0, keep_k=8)
    assert _noalloc(lib, None, 1, 256, 1024, [0], sp, fake)[0] == 1            # null logits
    assert _noalloc(lib, fake, 1, 256, 1024, [0], None, fake)[0] == 1          # null params
    rc, msg = _noalloc(lib, C.c_void_p(0x10004), 1, 256, 1024, [0], sp, fake)  # unaligned logits
    assert rc == 1 and "aligned" in msg
    assert _noalloc(lib, fake, 0, 256, 1024, [], sp, fake)[0] == 1             # empty batch
    assert _noalloc(lib, fake, 65, 256, 1024, list(range(65)), sp, fake)[0] == 1
    assert _noalloc(lib, fake, 1, 1025, 1024, [0], sp, fake)[0] == 1           # canvas too long
    assert _noalloc(lib, fake, 1, 256, 1024, [-1], sp, fake)[0] == 1           # negative request id
    assert _noalloc(lib, fake, 1, 4, 1024, [0], sp, fake)[0] == 1              # keep_k > n
    bad_t = B.sampler_params(temperature=-1.0, keep_k=1)
    assert _noalloc(lib, fake, 1, 256, 1024, [0], bad_t, fake)[0] == 1
    bad_mode = B.sampler_params(temperature=1.0, keep_k=1)
    bad_mode.keep_mode = 2
    rc, msg = _noalloc(lib, fake, 1, 256, 1024, [0], bad_mode, fake)
    assert rc == 1 and "keep_mode" in msg
    bad_stop = B.sampler_params(temperature=1.0, keep_k=1)
    bad_stop.stop_mode = 7
    rc, msg = _noalloc(lib, fake, 1, 256, 1024, [0], bad_stop, fake)
    assert rc == 1 and "stop_mode" in msg
    for budget in (-0.5, float("nan"), float("inf")):
        rc, msg = _noalloc(lib, fake, 1, 256, 1024, [0], B.sampler_params(entropy_budget=budget), fake)
        assert rc == 1 and "budget" in msg
    # 64 canvases of 256 over 262144 tokens exceed the fixed scratch: capacity error, nothing launched
    rc, msg = _noalloc(lib, fake, 64, 256, 262144, list(range(64)), sp, fake)
    assert rc == 4 and "scratch" in msg


def test_bench_algorithmic_counts_match_brute_force():
    """The flop and byte formulas behind bench.py's rooflines, against direct
    counts on tiny shapes."""
    import bench
    model = dict(n_heads=2, head_dim=4, n_layers=3, d_model=8, d_ff=6)
    prompt, canvas, steps = 5, 3, 2
    pairs = 0
    for _ in range(steps):                      # canvas step: every query sees prompt + canvas
        pairs += canvas * (prompt + canvas)
    pairs += sum(prompt + i + 1 for i in range(canvas))     # causal hand-off
    want = 2 * 2 * model["head_dim"] * model["n_heads"] * pairs * model["n_layers"]   # QK^T + PV, 2 flops/MAC
    assert bench.attention_flops(model, 1, canvas, [(prompt, steps)]) == want
    assert bench.attention_flops(model, 2, canvas, [(prompt, steps), (prompt + canvas, 1)]) == 2 * (
        want + 4 * model["head_dim"] * model["n_heads"] * model["n_layers"] *
        (1 * canvas * (prompt + 2 * canvas) + sum(prompt + canvas + i + 1 for i in range(canvas))))
    # gate+up bytes: touched experts' two [F, d] bf16 matrices, the rows read, the bf16 SwiGLU rows written
    d, f = model["d_model"], model["d_ff"]
    assert bench.moe_up_bytes(model, 10, 3) == 3 * 2 * f * d * 2 + 10 * d * 2 + 10 * f * 2


def test_bench_pass_cost_matches_weight_tensors_and_product_shapes():
    """bench.pass_cost's bytes against the sizes of the synthetic weight tensors
    (bf16) plus the KV traffic, and its flops against the products of one layer
    written out shape by shape."""
    import bench
    from discrete_text_diffusion_b200 import synth
    model = dict(n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, n_experts=6, top_k=2, d_ff=32,
                 vocab=100, canvas=8, rope_base=10000.0, rms_eps=1e-6)
    w = synth.make_weights(model, seed=0, dtype="bf16", router_bias=True)
    L0 = w["layers"][0]
    touched = 3
    attn = sum(L0[k].numel() for k in ("wq", "wk", "wv", "wo")) * 2
    router = L0["router_w"].numel() * 2
    expert = (L0["w_gate"][0].numel() + L0["w_up"][0].numel() + L0["w_down"][0].numel()) * 2
    B, n, P = 2, model["canvas"], 11
    kv = 2 * model["n_kv_heads"] * model["head_dim"] * 2           # K and V bf16 per position
    want_b = model["n_layers"] * (attn + router + touched * expert + B * P * kv + 2 * B * n * kv) \
        + w["embed"].numel() * 2 + w["w_sc"].numel() * 2
    d, hq, hkv, hd, F, E, k, V = 64, 4, 2, 16, 32, 6, 2, 100
    T = B * n
    mm = lambda m_, k_, n_: 2 * m_ * k_ * n_
    layer = mm(T, d, hq * hd) + 2 * mm(T, d, hkv * hd) + mm(T, hq * hd, d) + mm(T, d, E) \
        + T * k * (2 * mm(1, d, F) + mm(1, F, d))
    attn_fl = B * hq * n * (P + n) * (mm(1, hd, 1) + mm(1, 1, hd))
    want_f = model["n_layers"] * (layer + attn_fl) + mm(T, d, V) + mm(T, d, d)
    b, f = bench.pass_cost(model, B, n, P, touched, causal=False, head=True, self_cond=True)
    assert b == want_b and f == want_f
    # the causal hand-off: query i sees P + i + 1 keys, no head, no self-conditioning
    b2, f2 = bench.pass_cost(model, B, n, P, touched, causal=True, head=False, self_cond=False)
    attn_c = B * hq * sum(P + i + 1 for i in range(n)) * (mm(1, hd, 1) + mm(1, 1, hd))
    assert f2 == model["n_layers"] * (layer + attn_c)
    assert b2 == want_b - w["embed"].numel() * 2 - w["w_sc"].numel() * 2


def test_bench_block_roofline_sums_pass_bounds():
    import bench
    model = dict(n_layers=1, d_model=64, n_heads=2, n_kv_heads=1, head_dim=64, n_experts=4, top_k=1, d_ff=64,
                 vocab=64, canvas=4)
    peaks = {"hbm_gbs": 1.0, "bf16_tflops": 1.0, "bf16_tflops_sustained": 1.0}
    r = bench.block_roofline(model, 1, 4, [(10, 3)], 2, 1000.0, peaks)
    want = 0.0
    for t in (1, 2, 3):
        b, f = bench.pass_cost(model, 1, 4, 10, 2, False, True, t > 1)
        want += max(b / 1e9, f / 1e12)
    b, f = bench.pass_cost(model, 1, 4, 10, 2, True, False, False)
    want += max(b / 1e9, f / 1e12)
    assert abs(r["bound_ms_per_block"] - round(want * 1e3, 3)) < 1e-6
    assert abs(r["frac"] - round(want / 1.0, 4)) < 1e-6
