"""Pins for the oracle's MXFP4 on 16-element blocks (MXFP4_16): E2M1 elements
and E8M0 power-of-two scales, one scale per 16 consecutive K elements.

The microscaling form of "Portable FP4 quantization (TransFP4)" §1.1 Eq.(1)
leaves the block size G open (smaller G: more scale metadata, less outlier
spill); "4.5 FP8 and NVFP4/MXFP4" §3.3 gives the two formats that differ in
block size AND scale encoding.  E8M0 scales on 16-element blocks separate the
two effects and are the 16-element scale vector the block-scaled MMA also
takes with E8M0 scales.

What fixes it, independently of the oracle's own arithmetic:
  - scale bytes: a brute-force search over all 254 finite E8M0 scales per
    16-block (CEIL rule) and floor(log2 amax) - 2 (FLOOR rule);
  - elements: the brute-force nearest E2M1 point of x / 2^e, both tie rules;
  - against MXFP4 on 32-element blocks: no element's error is larger (the
    16-block exponent is at most the 32-block one, and below the block max
    the finer grid contains every point of the coarser one), and where both
    halves of a unit take the unit's exponent the codes are identical.
"""
import math

import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _x(rows, cols, seed, outliers=True):
    rng = np.random.default_rng(seed)
    v = rng.laplace(0, 1.0, (rows, cols)).astype(np.float32)
    if outliers:
        v[rng.random((rows, cols)) < 0.02] *= 40
    # a spread of row magnitudes, tiny and large, to cover many exponents
    v *= np.float32(2.0) ** rng.integers(-60, 60, (rows, 1)).astype(np.float32)
    v[0, :16] = 0.0  # one all-zero block
    return inputs.f32_to_bf16_bits(v)


def _codes(q):
    return np.stack([q & 15, q >> 4], -1).reshape(q.shape[0], -1).astype(int)


def _brute_e2m1(a, tie):
    """Nearest magnitude code of a >= 0 on the grid, saturating at 6."""
    if a >= 6.0:
        return 7
    d = np.abs(GRID - a)
    best = np.flatnonzero(d == d.min())
    if len(best) == 1:
        return int(best[0])
    lo, hi = int(best[0]), int(best[1])
    return hi if tie == 1 else (lo if lo % 2 == 0 else hi)


@pytest.mark.parametrize("rule", [0, 1])
def test_scale_bytes_by_brute_force(orc, rule):
    x = _x(16, 512, 1 + rule)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    _, s, g = orc.quantize(x, orc.MXFP4_16, mx_rule=rule)
    assert g == 1.0 and s.shape == (16, 32)
    scales = np.array([2.0 ** (b - 127) for b in range(255)])
    amax = np.abs(xf).reshape(16, 32, 16).max(-1)
    for r in range(16):
        for kb in range(32):
            a = amax[r, kb]
            if a == 0.0:
                want = 0
            elif rule == 0:
                want = int(np.flatnonzero(a / scales <= 6.0)[0])
            else:
                want = max(0, min(254, math.floor(math.log2(a)) - 2 + 127))
            assert int(s[r, kb]) == want, (r, kb, a)


@pytest.mark.parametrize("tie", [0, 1])
def test_elements_by_brute_force(orc, tie):
    x = _x(8, 256, 3)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    q, s, _ = orc.quantize(x, orc.MXFP4_16, tie=tie)
    c = _codes(q)
    for r in range(8):
        for i in range(256):
            e = int(s[r, i // 16]) - 127
            v = xf[r, i] / 2.0 ** e  # exact: a power-of-two quotient of a bf16 value
            want = _brute_e2m1(abs(v), tie) | (8 if math.copysign(1.0, v) < 0 else 0)
            assert c[r, i] == want, (r, i, v)
    # dequantization is code value times 2^e, exactly
    xh = orc.dequantize(q, s, 1.0, orc.MXFP4_16).astype(np.float64)
    mag = GRID[c & 7] * np.where(c & 8, -1.0, 1.0)
    d = np.repeat(2.0 ** (s.astype(np.float64) - 127), 16, axis=1)
    assert np.array_equal(xh, mag * d)


@pytest.mark.parametrize("tie", [0, 1])
@pytest.mark.parametrize("hk", [0, 32])
def test_error_never_above_32_element_blocks(orc, tie, hk):
    x = _x(16, 1024, 5 + hk + tie)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    q16, s16, _ = orc.quantize(x, orc.MXFP4_16, tie=tie, hadamard_k=hk)
    q32, s32, _ = orc.quantize(x, orc.MXFP4, tie=tie, hadamard_k=hk)
    # the 16-block exponents never exceed the 32-block one of their unit
    assert np.all(s16.reshape(16, -1, 2).max(-1) == s32)
    if hk == 0:
        e16 = np.abs(xf - orc.dequantize(q16, s16, 1.0, orc.MXFP4_16))
        e32 = np.abs(xf - orc.dequantize(q32, s32, 1.0, orc.MXFP4))
        assert np.all(e16 <= e32)
        assert e16.sum() < e32.sum()
    else:
        # elementwise in the rotated domain, where the blocks are quantized
        y = np.stack([orc.fwht(np.float32(xf[r]), hk) for r in range(16)]).astype(np.float64)
        e16 = np.abs(y - orc.dequantize(q16, s16, 1.0, orc.MXFP4_16))
        e32 = np.abs(y - orc.dequantize(q32, s32, 1.0, orc.MXFP4))
        assert np.all(e16 <= e32)
    same = np.repeat(s16 == np.repeat(s32, 2, axis=1), 16, axis=1)
    assert same.any() and (~same).any()
    assert np.array_equal(_codes(q16)[same], _codes(q32)[same])


def test_sign_symmetry_and_power_of_two_scaling(orc):
    x = _x(8, 256, 9)
    q, s, _ = orc.quantize(x, orc.MXFP4_16)
    qn, sn, _ = orc.quantize(x ^ np.uint16(0x8000), orc.MXFP4_16)
    assert np.array_equal(_codes(qn), _codes(q) ^ 8) and np.array_equal(s, sn)
    xs = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(x) * np.float32(2.0 ** -3))
    q3, s3, _ = orc.quantize(xs, orc.MXFP4_16)
    nz = s > 0
    assert np.array_equal(q3, q) and np.array_equal(s3.astype(int)[nz], s.astype(int)[nz] - 3)


def test_shape_rules(orc):
    with pytest.raises(ValueError):
        orc.quantize(np.zeros((2, 40), np.uint16), orc.MXFP4_16)  # not a multiple of 16
    q, s, _ = orc.quantize(np.zeros((2, 48), np.uint16), orc.MXFP4_16)
    assert q.shape == (2, 24) and s.shape == (2, 3) and not s.any()
