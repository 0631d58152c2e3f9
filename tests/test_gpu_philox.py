"""The device Philox4x32-10 equals the oracle's and cuRAND's (called, not read)."""
import numpy as np
import pytest
import torch

from oracle import dg_oracle as O


@pytest.mark.gpu
def test_device_philox_matches_oracle_and_curand(dg):
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="fp32", max_batch=1, max_ctx=64)
    rng = np.random.default_rng(0)
    n = 4096
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2**32, size=(n, 2), dtype=np.uint64).astype(np.uint32)
    ctr[:3] = [[0, 0, 0, 0], [0xFFFFFFFF] * 4, [0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344]]
    key[:3] = [[0, 0], [0xFFFFFFFF] * 2, [0xA4093822, 0x299F31D0]]
    dc = torch.from_numpy(ctr.view(np.int32)).cuda()
    dk = torch.from_numpy(key.view(np.int32)).cuda()
    out = torch.zeros((n, 4), dtype=torch.int32, device="cuda")
    out_cr = torch.zeros((n, 4), dtype=torch.int32, device="cuda")
    dg.dg_selftest_philox(h, dc, dk, out, out_cr)
    dg.dg_synchronize(h)
    got = out.cpu().numpy().view(np.uint32)
    want = O.philox4x32_10(ctr, key)
    assert np.array_equal(got, want)
    assert np.array_equal(out_cr.cpu().numpy().view(np.uint32), want)
    h.close()
