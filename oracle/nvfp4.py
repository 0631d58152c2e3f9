"""NVFP4 weights: element and scale codes, quantisation, dequantisation (TEST INFRASTRUCTURE).

This module is test infrastructure, not product code.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The CUDA library shares no code with it.

What the pages fix:
  [P2] DiffusionGemma overview (youleyou.com), "推荐的部署与优化方案": the model
       is tuned for NVFP4, a 4-bit floating-point format, on Blackwell and
       Hopper, with accuracy close to lossless.
  [P4] gitcode.csdn.net article, "MoE 26B参数架构分析", the NVFP4 bullet: the
       format is used to cut the weights' memory footprint.
The pages give no bit-level definition, so the format is taken from its
public definitions:
  [OCP-MX] OCP Microscaling Formats (MX) Specification v1.0, the FP4 E2M1
       element type: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit; no
       infinities or NaN; largest magnitude 6.
  [OFP8] OCP 8-bit Floating Point Specification (OFP8), E4M3: 1 sign, 4
       exponent bits with bias 7, 3 mantissa bits; S.1111.111 is NaN; largest
       finite magnitude 448; no infinities.
  [NVFP4] NVIDIA's published NVFP4 layout (PTX ISA, block-scaled MMA with a
       16-element scale vector): E2M1 elements, one E4M3 scale per 16
       consecutive elements, and one fp32 scale per tensor.

Readings of points those sources leave to the user (each is a named reading):
  R-fp4-block  a weight matrix [out, in] is scaled in blocks of 16 consecutive
               elements along `in`, the contraction dimension; `in` must be a
               multiple of 16.
  R-fp4-scale  per-tensor decode scale g = fp32(amax|W| / (6 * 448)) (1.0 for an
               all-zero tensor), so the largest block scale lands on E4M3's top
               value; block scale s_b = E4M3(amax_b / (6 g)); element code
               q = E2M1(w / (s_b g)); a block whose scale rounds to 0 has all
               codes 0.  Dequantised w = E2M1value(q) * E4M3value(s_b) * g.
  R-fp4-round  both encoders round to nearest with ties to the even code
               (mantissa bit 0) and saturate at the largest finite magnitude,
               as a round-to-nearest, saturate-to-finite conversion does.
  R-fp4-pack   two elements per byte: element 2j in bits 0-3, element 2j+1 in
               bits 4-7 of byte j of its row.
  R-fp4-act    weights only: activations stay in the model's activation type
               and the products are taken against the dequantised weights.

Parity pins: ``tests/test_oracle_nvfp4.py`` pins every public function here
against torch's float8_e4m3fn conversion, the OCP E2M1 value table, brute
force and exact round trips.  Parity unpinned: none.
"""
from __future__ import annotations

import numpy as np

BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0


# ----------------------------------------------------------------------------
# Element and scale codes ([OCP-MX], [OFP8]).
# ----------------------------------------------------------------------------

def e2m1_decode(codes):
    """FP4 E2M1 codes (0..15) -> float64 values.  Exponent 0 is subnormal:
    m * 0.5; otherwise 2^(e-1) * (1 + m/2)."""
    c = np.asarray(codes).astype(np.int64)
    if c.size and (c.min() < 0 or c.max() > 15):
        raise ValueError("E2M1 codes are 4-bit")
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, e - 1))
    return sign * mag


def e4m3_decode(codes):
    """E4M3 codes (0..255) -> float64 values; S.1111.111 -> NaN.  Exponent 0
    is subnormal: (m/8) * 2^-6; otherwise 2^(e-7) * (1 + m/8)."""
    c = np.asarray(codes).astype(np.int64)
    if c.size and (c.min() < 0 or c.max() > 255):
        raise ValueError("E4M3 codes are 8-bit")
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 0xF) & (m == 0x7), np.nan, mag)
    return sign * mag


def _round_to_codes(x, codes):
    """Round |x| to the nearest of the non-negative values of `codes` (given
    as (code, value) pairs in increasing value), ties to the even code,
    saturating at the largest.  Returns the chosen codes."""
    cv = np.array([v for _, v in codes])
    cc = np.array([c for c, _ in codes])
    a = np.abs(np.asarray(x, dtype=np.float64))
    flat = a.reshape(-1, 1)
    d = np.abs(cv[None, :] - flat)                         # distance to every candidate value
    nearest = d == d.min(axis=1, keepdims=True)            # one candidate, or two on a tie
    even_nearest = nearest & (cc[None, :] % 2 == 0)
    pick = np.where(even_nearest.any(axis=1), np.argmax(even_nearest, axis=1), np.argmax(nearest, axis=1))
    out = cc[pick]
    out = np.where(flat[:, 0] >= cv[-1], cc[-1], out)      # saturate at the largest value
    return out.reshape(a.shape)


def e2m1_encode(x):
    """float -> E2M1 code, round to nearest, ties to the even code, saturating
    at 6 (R-fp4-round).  The sign bit follows the sign of x (-0.0 -> code 8)."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no E2M1 code")
    pos = [(c, float(e2m1_decode(c))) for c in range(8)]
    mag = _round_to_codes(x, pos)
    return (mag | np.where(np.signbit(x), 0x8, 0)).astype(np.uint8)


def e4m3_encode_nonneg(x):
    """float >= 0 -> E4M3 code, round to nearest, ties to the even code,
    saturating at 448 (R-fp4-round).  Used for block scales, which are >= 0."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any() or (x < 0).any():
        raise ValueError("block scales are finite and >= 0")
    pos = [(c, float(e4m3_decode(c))) for c in range(0x7F)]      # 0 .. 448
    return _round_to_codes(x, pos).astype(np.uint8)


# ----------------------------------------------------------------------------
# Quantisation of a weight matrix ([NVFP4], R-fp4-block, R-fp4-scale).
# ----------------------------------------------------------------------------

def quantize(w):
    """w [rows, K] (K a multiple of 16) -> dict(codes uint8 [rows, K],
    scales uint8 [rows, K/16] (E4M3 codes), g float (an fp32 value))."""
    w = np.asarray(w, dtype=np.float64)
    if w.ndim != 2 or w.shape[1] % BLOCK:
        raise ValueError("quantize wants [rows, K] with K a multiple of 16")
    rows, k = w.shape
    amax = float(np.max(np.abs(w))) if w.size else 0.0
    g = float(np.float32(amax / (E2M1_MAX * E4M3_MAX))) if amax > 0 else 1.0
    blocks = w.reshape(rows, k // BLOCK, BLOCK)                   # [rows, block, element]
    amax_b = np.max(np.abs(blocks), axis=2) if w.size else np.zeros((rows, k // BLOCK))
    scales = e4m3_encode_nonneg(amax_b / (E2M1_MAX * g)).astype(np.uint8)
    s = e4m3_decode(scales)[..., None]                             # the scale each block decodes with
    codes = np.where(s > 0, e2m1_encode(blocks / (np.where(s > 0, s, 1.0) * g)), 0)
    return dict(codes=codes.reshape(rows, k).astype(np.uint8), scales=scales, g=g)


def dequantize(q):
    """The float64 matrix a quantised weight stands for:
    E2M1value(code) * E4M3value(block scale) * g."""
    codes, scales, g = q["codes"], q["scales"], q["g"]
    rows, k = codes.shape
    if scales.shape != (rows, k // BLOCK):
        raise ValueError("one scale per 16 elements of a row")
    s = np.repeat(e4m3_decode(scales), BLOCK, axis=1)
    return e2m1_decode(codes) * s * g


# ----------------------------------------------------------------------------
# Storage (R-fp4-pack).
# ----------------------------------------------------------------------------

def pack(codes):
    """[rows, K] codes -> [rows, K/2] bytes, element 2j in the low nibble."""
    c = np.asarray(codes).astype(np.uint8)
    if c.shape[-1] % 2:
        raise ValueError("an even number of elements per row")
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack(packed):
    """[rows, K/2] bytes -> [rows, K] codes."""
    p = np.asarray(packed).astype(np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
