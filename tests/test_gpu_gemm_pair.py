"""The split-K dense product on CTA pairs (tcgen05 cta_group::2: two SMs per
256-row weight tile, each holding 128 weight rows and half of the token tile)
against a float64 matmul of the same bf16 operands, through the C ABI: the
QKV, O and self-conditioning shapes of the full-width layer, plus ragged M
(a pair whose second half is past the last weight row), ragged T (a token
tile whose second half is past the last token), one-chunk K slices and the
narrow token tiles."""
import ctypes as C

import pytest
import torch

from tests._util import max_abs_rel, to_np

DG_EINVAL = 1


def _run(dg, T, Mr, K, ntile, ksplit, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((T, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((Mr, K), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    part = torch.full((ksplit, T, Mr), float("nan"), device="cuda")
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="bf16", max_batch=1, max_ctx=64)
    dg.dg_selftest_gemm_pair(h, x, w, part, ntile)
    dg.dg_synchronize(h)
    h.close()
    assert not torch.isnan(part).any(), "a slice element was not written"
    ref = x.double().cpu() @ w.double().cpu().T
    return max_abs_rel(to_np(part.double().sum(0)), ref.numpy())


@pytest.mark.gpu
@pytest.mark.parametrize("T,Mr,K,ntile,ksplit", [
    (256, 8192, 2816, 256, 2),     # Q|K|V at batch 1
    (256, 2816, 4096, 256, 3),     # O projection
    (256, 2816, 2816, 256, 2),     # self-conditioning
    (200, 300, 192, 256, 3),       # ragged T inside the pair's tile, ragged M inside the second pair
    (130, 256, 128, 128, 2),       # second token tile holds 2 rows: the second CTA's half is empty
    (37, 512, 640, 64, 1),
    (64, 384, 256, 64, 4),         # one 64-column chunk per slice
    (96, 512, 320, 128, 2),        # 5 chunks: the last stage of two chunks runs past K
    (1, 128, 64, 64, 1),
])
def test_pair_gemm_slices_sum_to_float64_matmul(dg, T, Mr, K, ntile, ksplit):
    err = _run(dg, T, Mr, K, ntile, ksplit, seed=T * 11 + Mr)
    assert err < 1e-3, err


@pytest.mark.gpu
def test_pair_gemm_rejects_bad_tiles(dg):
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    part = torch.zeros((4, 64, 128), device="cuda")
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="bf16", max_batch=1, max_ctx=64)
    L = dg.lib()
    args = lambda nt, ks: (h.ptr, C.c_void_p(x.data_ptr()), C.c_void_p(w.data_ptr()), 64, 128, 128, nt, ks,  # noqa
                           C.c_void_p(part.data_ptr()))
    assert L.dg_selftest_gemm_pair(*args(96, 1)) == DG_EINVAL     # token tile not 64 / 128 / 256
    assert L.dg_selftest_gemm_pair(*args(64, 3)) == DG_EINVAL     # 3 slices of 2 chunks
    assert L.dg_selftest_gemm_pair(*args(64, 0)) == DG_EINVAL
    h.close()
