"""Pins of the NVFP4 oracle (oracle/nvfp4.py) against things other than itself:
the OCP E2M1 value table, torch's float8_e4m3fn conversion (a library
routine), brute force, bounds that follow from the format, and exact round
trips of weights built from codes."""
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4 as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e2m1_values.txt")) if not ln.startswith("#")]
    return {int(c): float(v) for c, v in rows}


def test_e2m1_decode_matches_the_ocp_table():
    table = _e2m1_table()
    got = F.e2m1_decode(np.arange(16))
    assert len(table) == 16
    for c in range(16):
        assert got[c] == table[c] and np.signbit(got[c]) == np.signbit(table[c]), c


def test_e4m3_decode_matches_torch_float8_e4m3fn():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = F.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.nanmax(got) == 448.0 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])


def test_e4m3_encode_matches_torch_rounding():
    vals = F.e4m3_decode(np.arange(0x7F))                      # 0 .. 448, increasing
    mids = (vals[:-1] + vals[1:]) / 2                          # every tie
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(0, 448, 4000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 4000)),
                           [448.0, 449.0, 463.9, 1e-9, 2.0 ** -10, 2.0 ** -10 * 1.0001]])
    x = np.concatenate([vals, mids, rand])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # float32 inputs on both sides: the tie values are exact in float32
    got = F.e4m3_encode_nonneg(x.astype(np.float32).astype(np.float64))
    assert np.array_equal(got, want)
    assert F.e4m3_encode_nonneg([1e6]).tolist() == [0x7E]       # saturates (torch gives NaN there)
    with pytest.raises(ValueError):
        F.e4m3_encode_nonneg([-1.0])


def test_e2m1_encode_is_nearest_with_ties_to_even_by_brute_force():
    table = _e2m1_table()
    vals = np.array([table[c] for c in range(16)])
    x = np.concatenate([np.linspace(-8, 8, 4097), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 6.0, 6.5, -100.0]])
    got = F.e2m1_encode(x)
    for xi, c in zip(x, got):
        d = np.abs(vals - xi)
        # the chosen value is at least as near as any other
        assert d[c] == d.min() or abs(xi) > 6.0, xi
        if abs(xi) > 6.0:
            assert vals[c] == np.sign(xi) * 6.0
        ties = [k for k in range(16) if d[k] == d.min() and np.signbit(vals[k]) == np.signbit(xi)]
        if len(ties) > 1 and abs(xi) <= 6.0:
            assert c % 2 == 0, xi                                  # the even code wins a tie
        assert bool(c & 8) == bool(np.signbit(xi))
    assert F.e2m1_encode([0.25, 0.75, 2.5, 5.0]).tolist() == [0, 2, 4, 6]
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(np.arange(16))), np.arange(16))


def _weights_from_codes(rng, rows, k, g):
    """A weight matrix that NVFP4 represents exactly: random codes, every block
    holding a +-6 element, random block scales with the top one at 448."""
    codes = rng.integers(0, 16, (rows, k)).astype(np.uint8)
    for r in range(rows):
        for b in range(k // 16):
            codes[r, b * 16 + rng.integers(0, 16)] = rng.choice([7, 15])
    scales = rng.integers(0x20, 0x7F, (rows, k // 16)).astype(np.uint8)
    scales[rng.integers(0, rows), rng.integers(0, k // 16)] = 0x7E
    w = F.e2m1_decode(codes) * np.repeat(F.e4m3_decode(scales), 16, axis=1) * g
    return w, codes, scales


@pytest.mark.parametrize("seed", range(3))
def test_quantize_reproduces_weights_built_from_codes(seed):
    rng = np.random.default_rng(seed)
    g = float(np.float32(rng.uniform(1e-5, 1e-3)))
    w, codes, scales = _weights_from_codes(rng, 5, 64, g)
    q = F.quantize(w)
    assert q["g"] == g
    assert np.array_equal(q["scales"], scales)
    # -0 and +0 encode the same value; compare values there, codes elsewhere
    nz = F.e2m1_decode(codes) != 0
    assert np.array_equal(q["codes"][nz], codes[nz])
    assert np.array_equal(F.dequantize(q), w)


def test_quantize_error_bound_and_structure():
    rng = np.random.default_rng(7)
    w = rng.standard_normal((24, 96)) * rng.uniform(0.001, 0.1, (24, 1))
    w[3, 16:32] = 0.0                                      # an all-zero block
    q = F.quantize(w)
    assert q["codes"].shape == w.shape and q["scales"].shape == (24, 6)
    assert q["g"] == np.float32(np.abs(w).max() / 2688.0)
    deq = F.dequantize(q)
    s = np.repeat(F.e4m3_decode(q["scales"]), 16, axis=1) * q["g"]
    # each element lands within one grid step of the 4 -> 6 gap's half (1.0) of its block's scale,
    # and small elements within half the finest step (0.25)
    err = np.abs(deq - w)
    assert (err <= 1.0 * s + 1e-15).all()
    small = np.abs(w) <= 2.0 * s
    assert (err[small] <= 0.25 * s[small] + 1e-15).all()
    assert (q["scales"][3, 1] == 0) and (deq[3, 16:32] == 0).all()
    # every block's largest element uses the top of the E2M1 range, up to the scale's rounding
    top = np.abs(F.e2m1_decode(q["codes"])).reshape(24, 6, 16).max(axis=2)
    assert ((top >= 4.0) | (q["scales"] == 0)).all()
    # the tensor's largest element sits in a block whose scale is E4M3's top value
    r, c = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert q["scales"][r, c // 16] == 0x7E
    with pytest.raises(ValueError):
        F.quantize(np.zeros((2, 24)))
    z = F.quantize(np.zeros((2, 32)))
    assert z["g"] == 1.0 and not z["codes"].any() and not z["scales"].any()


def test_pack_nibble_order_and_round_trip():
    assert F.pack(np.array([[1, 2, 15, 0]])).tolist() == [[0x21, 0x0F]]
    c = np.random.default_rng(3).integers(0, 16, (7, 48)).astype(np.uint8)
    p = F.pack(c)
    assert p.shape == (7, 24) and p.dtype == np.uint8
    assert np.array_equal(F.unpack(p), c)
    with pytest.raises(ValueError):
        F.pack(np.zeros((1, 3), dtype=np.uint8))
