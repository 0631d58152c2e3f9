"""dg_sample_noalloc against dg_sample, through the C ABI.

dg_sample_noalloc runs the same sampler kernels as dg_sample but keeps its
per-call scratch in a fixed device array instead of a handle's workspace.
Its outputs must equal dg_sample's on the same logits, request ids and
Philox counters, call after call.  This file is named to be collected last,
so the entry point is also exercised after every other test has run in the
same process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from discrete_text_diffusion_b200 import synth
from tests._util import to_np

W = synth.WORKLOADS["sampler"]
DG_ECAPACITY = 4


def _outs(B, n):
    dev = "cuda"
    return dict(x_hat=torch.zeros((B, n), dtype=torch.int32, device=dev),
                pmax=torch.zeros((B, n), device=dev), entropy=torch.zeros((B, n), device=dev),
                keep=torch.zeros((B, n), dtype=torch.int32, device=dev),
                mean_entropy=torch.zeros(B, device=dev), stop=torch.zeros(B, dtype=torch.int32, device=dev))


def _via_handle(dg, logits, req, step, sp):
    B, n, V = logits.shape
    h = dg.dg_create(dict(vocab=V, canvas=n), None, dtype="fp32", max_batch=max(req) + 1, max_ctx=max(64, n))
    outs = _outs(B, n)
    canvas = torch.full((B, n), -1, dtype=torch.int32, device="cuda")
    dg.dg_sample(h, logits, req, step, sp, canvas, dg.step_out(**outs))
    dg.dg_synchronize(h)
    h.close()
    outs["canvas"] = canvas
    return {k: to_np(v) for k, v in outs.items()}


def _via_noalloc(dg, logits, req, step, sp, with_outputs=True):
    B, n, V = logits.shape
    outs = _outs(B, n) if with_outputs else {}
    canvas = torch.full((B, n), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    dg.dg_sample_noalloc(logits, req, step, sp, canvas, dg.step_out(**outs), stream=stream)
    stream.synchronize()
    outs["canvas"] = canvas
    return {k: to_np(v) for k, v in outs.items()}


def _same(a, b):
    for k in a:
        if a[k].dtype.kind == "f":
            # identical kernels on identical inputs: the tolerance only allows for nothing
            assert np.allclose(a[k], b[k], rtol=1e-6, atol=1e-7), k
        else:
            assert np.array_equal(a[k], b[k]), k


@pytest.mark.gpu
def test_noalloc_sampler_matches_dg_sample_two_calls_in_a_row(dg):
    B, n, V = 2, W["canvas"], W["vocab"]
    logits, _, _ = synth.peaked_logits(B, n, V, seed=W["seed"] + 91, peak_max=W["peak_max"])
    logits = logits.cuda()
    req = [3, 1]
    sp = dg.sampler_params(temperature=W["temperature"], keep_k=128, stop_threshold=W["stop_threshold"],
                           seed=77, block=5)
    for step in (1, 2):   # two calls in a row reuse the same scratch
        want = _via_handle(dg, logits, req, step, sp)
        got = _via_noalloc(dg, logits, req, step, sp)
        _same(got, want)
    # without output buffers, x_hat / pmax / entropy go to the scratch; the canvas is unchanged
    got = _via_noalloc(dg, logits, req, 2, sp, with_outputs=False)
    assert np.array_equal(got["canvas"], want["canvas"])


@pytest.mark.gpu
def test_noalloc_sampler_leaves_free_device_memory_unchanged(dg):
    """The property the entry point exists for: once the device is set up (the
    first call), calls take no device memory.  Free memory is read with
    cudaMemGetInfo around repeated calls, with every output buffer made first."""
    B, n, V = 2, W["canvas"], W["vocab"]
    logits, _, _ = synth.peaked_logits(B, n, V, seed=W["seed"] + 92, peak_max=W["peak_max"])
    logits = logits.cuda()
    sp = dg.sampler_params(temperature=W["temperature"], keep_k=64, stop_threshold=W["stop_threshold"], seed=5)
    outs = _outs(B, n)
    canvas = torch.zeros((B, n), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    o = dg.step_out(**outs)
    dg.dg_sample_noalloc(logits, [0, 1], 1, sp, canvas, o, stream=stream)     # set-up call
    stream.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for step in range(2, 7):
        dg.dg_sample_noalloc(logits, [0, 1], step, sp, canvas, o, stream=stream)
        dg.dg_sample_noalloc(logits, [0, 1], step, sp, canvas, None, stream=stream)
    stream.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes across calls"


@pytest.mark.gpu
def test_noalloc_sampler_argmax_ragged_vocab(dg):
    B, n, V = 3, 37, 5001
    g = torch.Generator().manual_seed(5)
    logits = torch.randn((B, n, V), generator=g).cuda()
    sp = dg.sampler_params(temperature=0.0, keep_k=9, stop_threshold=0.5, seed=2)
    _same(_via_noalloc(dg, logits, [0, 1, 2], 4, sp), _via_handle(dg, logits, [0, 1, 2], 4, sp))


@pytest.mark.gpu
def test_noalloc_sampler_rejects_requests_beyond_its_scratch(dg):
    # 64 canvases of 256 over 262144 tokens need ~25 MB of chunk partials; the scratch is 8 MiB.
    # The size check runs on the host before anything is launched, so no logits are read.
    B, n, V = 64, 256, 262144
    fake = torch.zeros(16, device="cuda")     # pointer only
    canvas = torch.zeros(16, dtype=torch.int32, device="cuda")
    sp = dg.sampler_params(temperature=1.0, keep_k=8)
    err = C.create_string_buffer(256)
    rc = dg.lib().dg_sample_noalloc(C.c_void_p(fake.data_ptr()), B, n, V, (C.c_int * B)(*range(B)), 1,
                                    C.byref(sp), C.c_void_p(canvas.data_ptr()), None, None, err, 256)
    assert rc == DG_ECAPACITY
    assert b"scratch" in err.value
