"""Pins for the CPU oracle: what the pages print and what mathematics fixes.

Every check here compares the oracle with something other than itself: values
printed on the pages (tests/golden/), a brute-force search, an independent
library routine (torch's float8 cast, scipy's Hadamard matrix, numpy's fp64
matmul), closed forms, or invariants that a dropped term, wrong sign, wrong
index or transposed operand would break.
"""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    rows = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    return rows


def f32(x):
    return np.float32(x)


def bits_f32(u):
    return np.array([u], np.uint32).view(np.float32)[0]


GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def brute_e2m1(v, tie):
    """Independent nearest-point search over the 8 magnitudes."""
    a = abs(float(v))
    sign = 8 if math.copysign(1.0, float(v)) < 0 else 0
    if a >= 6.0:
        return sign | 7
    d = np.abs(GRID - a)
    best = np.flatnonzero(d == d.min())
    if len(best) == 1:
        c = int(best[0])
    else:  # exact midpoint between two neighbours
        lo, hi = int(best[0]), int(best[1])
        c = hi if tie == 1 else (lo if lo % 2 == 0 else hi)
    return sign | c


# ---------------------------------------------------------------- E2M1 -------
def test_e2m1_magnitude_set_matches_page(orc):
    g = golden("e2m1_magnitudes.txt")
    mags = [float(v) for v in g["magnitudes"][0]]
    assert [orc.e2m1_decode(c) for c in range(8)] == mags
    assert max(orc.e2m1_decode(c) for c in range(16)) == float(g["max"][0][0])
    vals = {(orc.e2m1_decode(c), math.copysign(1, orc.e2m1_decode(c)) if c else 1) for c in range(16)}
    assert len(vals) == int(g["codes"][0][0])
    for c in range(8):
        assert orc.e2m1_decode(c | 8) == -orc.e2m1_decode(c)
    # 0.5 is the only subnormal: exponent bits 00 with mantissa 1
    assert orc.e2m1_decode(0b0001) == 0.5 and orc.e2m1_decode(0b0111) == 6.0


def _e2m1_probe_values():
    vals = [bits_f32(np.uint32(b) << 16) for b in range(0, 1 << 16)]  # every bf16
    vals = [v for v in vals if np.isfinite(v)]
    pts = [0.0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7, 8]
    for p in pts:
        x = np.float32(p)
        for s in (1, -1):
            y = np.float32(s * x)
            vals += [y, np.nextafter(y, np.float32(np.inf)), np.nextafter(y, np.float32(-np.inf))]
    rng = np.random.default_rng(7)
    vals += list(rng.uniform(-7, 7, 20000).astype(np.float32))
    vals += [np.float32(np.inf), np.float32(-np.inf), np.float32(-0.0)]
    return vals


@pytest.mark.parametrize("tie", [0, 1])
def test_e2m1_encode_equals_bruteforce(orc, tie):
    for v in _e2m1_probe_values():
        assert orc.e2m1_encode(v, tie) == brute_e2m1(v, tie), (v, tie)


def test_e2m1_tie_table(orc):
    # ties: even code (default) / larger magnitude
    even = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    away = {0.25: 0.5, 0.75: 1.0, 1.25: 1.5, 1.75: 2.0, 2.5: 3.0, 3.5: 4.0, 5.0: 6.0}
    for v, want in even.items():
        assert orc.e2m1_decode(orc.e2m1_encode(v, 0)) == want
        assert orc.e2m1_decode(orc.e2m1_encode(-v, 0)) == -want
    for v, want in away.items():
        assert orc.e2m1_decode(orc.e2m1_encode(v, 1)) == want
    assert orc.e2m1_encode(-0.0, 0) == 8 and orc.e2m1_encode(-0.1, 0) == 8
    assert orc.e2m1_encode(1e30, 0) == 7 and orc.e2m1_encode(-6.5, 0) == 15


# ---------------------------------------------------------------- E4M3 -------
def test_e4m3_page_pins(orc):
    g = golden("e4m3_pins.txt")
    bits, val = g["bits"][0]
    assert orc.e4m3_decode(int(bits, 2)) == float(val)
    assert orc.e4m3_encode(float(val)) == int(bits, 2)
    mx = float(g["max"][0][0])
    assert max(orc.e4m3_decode(c) for c in range(0x7F)) == mx
    assert math.isnan(orc.e4m3_decode(0x7F))
    assert orc.e4m3_encode(1e9) == 0x7E and orc.e4m3_decode(0x7E) == mx
    for lo, hi, step in g["spacing"]:
        lo, hi, step = float(lo), float(hi), float(step)
        vals = sorted(orc.e4m3_decode(c) for c in range(0x7F) if lo <= orc.e4m3_decode(c) < hi)
        assert np.allclose(np.diff(vals), step) and vals[0] == lo
    ten = float(g["exact"][0][0])
    b = orc.e4m3_encode(ten)
    assert orc.e4m3_decode(b) == ten == 1.25 * 2 ** 3 and b == 0x52


def test_e4m3_encode_matches_torch_cast(orc):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    vals = [bits_f32(np.uint32(b) << 16) for b in range(0, 0x7F80)]  # all finite positive bf16
    vals = [v for v in vals if v < 448.0]
    vals += list(np.exp(rng.uniform(np.log(1e-4), np.log(447.9), 30000)).astype(np.float32))
    # midpoints between codes and their neighbours exercise the tie rule
    for c in range(0x7D):
        m = np.float32((orc.e4m3_decode(c) + orc.e4m3_decode(c + 1)) / 2)
        vals += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    t = torch.tensor(np.array(vals, np.float32))
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([orc.e4m3_encode(float(v)) for v in vals], np.uint8)
    bad = np.flatnonzero(ref != ours)
    assert bad.size == 0, [(vals[i], ref[i], ours[i]) for i in bad[:5]]


def test_e8m0(orc):
    assert orc.e8m0_decode(127) == 1.0
    assert orc.e8m0_decode(0) == 2.0 ** -127 and orc.e8m0_decode(254) == 2.0 ** 127
    assert math.isnan(orc.e8m0_decode(255))
    assert all(orc.e8m0_decode(b) != 10.0 for b in range(255))  # cannot store 10


# ---------------------------------------------------------------- MX scale ---
def _closed_form_ceil(amax):
    u = int(np.array([amax], np.float32).view(np.uint32)[0])
    ex, man = (u >> 23) & 0xFF, u & 0x7FFFFF
    if ex == 0:  # normalise a subnormal
        E = -126
        while man < 0x800000:
            man <<= 1
            E -= 1
        man &= 0x7FFFFF
    else:
        E = ex - 127
    e = E - 2 + (1 if man > 0x400000 else 0)
    return max(-127, min(127, e))


def test_mx_exponent_closed_form_and_bruteforce(orc):
    rng = np.random.default_rng(1)
    vals = list(np.exp(rng.uniform(np.log(1e-44), np.log(3e38), 4000)).astype(np.float32))
    vals += [np.float32(v) for v in (6, 6.0000005, 12, 1.5, 3, 0.375, 1e-45, 3.4e38, 7.99)]
    scales = np.array([2.0 ** (b - 127) for b in range(255)])
    for a in vals:
        a = np.float32(a)
        e = orc.mx_scale_exponent(a, 0)
        assert e == _closed_form_ceil(a), a
        ok = np.flatnonzero(float(a) / scales <= 6.0)
        assert e == max(-127, int(ok[0]) - 127), a
        ef = orc.mx_scale_exponent(a, 1)
        assert ef == max(-127, min(127, math.floor(math.log2(float(a))) - 2)), a
    assert orc.mx_scale_exponent(0.0, 0) == -127


def test_gptoss_worked_example(orc):
    g = golden("gptoss_worked_example.txt")
    xs = [float(v) for v in g["inputs"][0]]
    direct = [float(v) for v in g["direct"][0]]
    scaled = [float(v) for v in g["scaled"][0]]
    # direct conversion (scale 1): the page's 0.25 -> 0.5 is a tie broken away
    assert [orc.e2m1_decode(orc.e2m1_encode(v, 1)) for v in xs] == direct
    # one 32-element MXFP4 block (the four values padded with zeros)
    blk = np.zeros((1, 32), np.float32)
    blk[0, :4] = xs
    x = inputs.f32_to_bf16_bits(blk)
    for tie, want in ((1, scaled), (0, [1.0, 6.0, 1.0, 4.0])):
        q, s, _ = orc.quantize(x, orc.MXFP4, tie=tie)
        assert s[0, 0] == 127 - 4  # shared scale 2^-4
        codes = [(q[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(4)]
        assert [orc.e2m1_decode(c) for c in codes] == want
        xh = orc.dequantize(q, s, 1.0, orc.MXFP4)
        assert np.array_equal(xh[0, :4], np.array(want, np.float32) / 16)


def test_guide_scale_example(orc):
    g = golden("guide_scale_example.txt")
    for key, skey in (("block_a", "scale_a"), ("block_b", "scale_b")):
        blk = np.zeros((1, 16), np.float32)
        vals = [float(v) for v in g[key][0]]
        blk[0, :4] = vals
        x = inputs.f32_to_bf16_bits(blk)
        q, s, sg = orc.quantize(x, orc.NVFP4, gscale=1.0)
        assert sg == 1.0
        assert orc.e4m3_decode(int(s[0, 0])) == float(g[skey][0][0])
        xh = orc.dequantize(q, s, 1.0, orc.NVFP4)
        assert np.array_equal(xh[0, :4], np.array(vals, np.float32))
    # MXFP4 cannot use the scale 10: the same block is no longer exact
    blk = np.zeros((1, 32), np.float32)
    blk[0, :4] = [float(v) for v in g["block_b"][0]]
    x = inputs.f32_to_bf16_bits(blk)
    q, s, _ = orc.quantize(x, orc.MXFP4)
    xh = orc.dequantize(q, s, 1.0, orc.MXFP4)
    assert orc.e8m0_decode(int(s[0, 0])) == 16.0
    assert not np.array_equal(xh[0, :4], blk[0, :4])


# ---------------------------------------------------------------- tensors ----
def _rand_bf16(rows, cols, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    v = rng.laplace(0, scale, (rows, cols)).astype(np.float32)
    v[rng.random((rows, cols)) < 0.02] *= 30
    return inputs.f32_to_bf16_bits(v)


def _nibbles(q):
    lo = q & 0xF
    hi = q >> 4
    return np.stack([lo, hi], -1).reshape(q.shape[0], -1)


@pytest.mark.parametrize("fmt", [0, 1])
def test_sign_symmetry(orc, fmt):
    x = _rand_bf16(8, 256, 5)
    q1, s1, g1 = orc.quantize(x, fmt)
    q2, s2, g2 = orc.quantize(x ^ np.uint16(0x8000), fmt)
    assert np.array_equal(_nibbles(q2), _nibbles(q1) ^ 8)
    assert np.array_equal(s1, s2) and g1 == g2


@pytest.mark.parametrize("j", [-3, 5])
def test_power_of_two_scaling(orc, j):
    x = _rand_bf16(8, 256, 6)
    xs = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(x) * np.float32(2.0 ** j))
    qa, sa, _ = orc.quantize(x, 0)
    qb, sb, _ = orc.quantize(xs, 0)
    assert np.array_equal(qa, qb)
    assert np.array_equal(sb.astype(int), sa.astype(int) + j)
    qa, sa, ga = orc.quantize(x, 1)
    qb, sb, gb = orc.quantize(xs, 1)
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb) and gb == ga * 2.0 ** j


def test_nvfp4_global_scale_definition(orc):
    x = _rand_bf16(16, 512, 8)
    q, s, sg = orc.quantize(x, 1)
    amax = np.abs(inputs.bf16_bits_to_f32(x)).max()
    assert sg == np.float32(amax) / np.float32(6 * 448)
    assert int(s.max()) == 0x7E  # the largest block lands on the E4M3 maximum
    z = np.zeros((2, 32), np.uint16)
    q, s, sg = orc.quantize(z, 1)
    assert sg == 1.0 and not s.any() and not q.any()


@pytest.mark.parametrize("fmt", [0, 1])
def test_elements_round_to_nearest_grid_point(orc, fmt):
    """Each dequantized element is (up to the fp32 reciprocal) the nearest
    point of the block's grid d * {0, +-0.5, ..., +-6}."""
    x = _rand_bf16(16, 256, 9)
    q, s, sg = orc.quantize(x, fmt)
    xh = orc.dequantize(q, s, sg, fmt).astype(np.float64)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    block = 32 if fmt == 0 else 16
    for r in range(x.shape[0]):
        for kb in range(x.shape[1] // block):
            if fmt == 0:
                d = orc.e8m0_decode(int(s[r, kb]))
            else:
                d = float(np.float32(sg) * np.float32(orc.e4m3_decode(int(s[r, kb]))))
            grid = np.concatenate([GRID, -GRID]) * d
            for i in range(kb * block, (kb + 1) * block):
                best = np.min(np.abs(grid - xf[r, i]))
                # slack: one fp32 rounding of d * q in the dequantized value
                assert abs(xh[r, i] - xf[r, i]) <= best + 2.0 ** -23 * (abs(xf[r, i]) + 6 * d), (r, i)


def test_mx_value_idempotence(orc):
    x = _rand_bf16(8, 256, 10)
    q, s, _ = orc.quantize(x, 0)
    xh = orc.dequantize(q, s, 1.0, 0)
    q2, s2, _ = orc.quantize(inputs.f32_to_bf16_bits(xh), 0)
    xh2 = orc.dequantize(q2, s2, 1.0, 0)
    # x_hat values carry <= 2 significant bits, so they are exact in bf16
    assert np.array_equal(inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(xh)), xh)
    assert np.array_equal(xh, xh2)


def test_shape_validation(orc):
    x = np.zeros((2, 48), np.uint16)
    with pytest.raises(ValueError):
        orc.quantize(x, 0)  # 48 is not a multiple of the MX block
    with pytest.raises(ValueError):
        orc.quantize(np.zeros((2, 64), np.uint16), 0, hadamard_k=128)


def test_scale_counts_and_bits(orc):
    g = golden("scale_counts.txt")
    rows, cols = (int(v) for v in g["shape"][0])
    assert rows * (cols // 128) == int(g["group128"][0][0])
    x = np.zeros((rows, cols), np.uint16)
    _, s_mx, _ = orc.quantize(x, 0)
    _, s_nv, _ = orc.quantize(x, 1)
    assert s_mx.size == rows * cols // 32 and s_nv.size == rows * cols // 16
    assert 4 + 8 * s_mx.size / (rows * cols) == float(g["bits_mx"][0][0])
    assert 4 + 8 * s_nv.size / (rows * cols) == float(g["bits_nv"][0][0])


# ---------------------------------------------------------------- rotation ---
@pytest.mark.parametrize("k", [16, 32, 64, 128])
def test_fwht_equals_sylvester_matrix(orc, k):
    scipy_linalg = pytest.importorskip("scipy.linalg")
    H = scipy_linalg.hadamard(k).astype(np.float64) / math.sqrt(k)
    rng = np.random.default_rng(k)
    x = rng.standard_normal(4 * k).astype(np.float32)
    y = orc.fwht(x, k).astype(np.float64)
    ref = (x.astype(np.float64).reshape(4, k) @ H.T).reshape(-1)
    tol = 4 * k * 2.0 ** -24 * np.abs(x).reshape(4, k).sum(1).repeat(k)
    assert np.all(np.abs(y - ref) <= tol)
    back = orc.fwht(y.astype(np.float32), k)
    assert np.allclose(back, x, rtol=0, atol=1e-5 * np.abs(x).max())
    assert np.allclose(H @ H, np.eye(k), atol=1e-12)


@pytest.mark.parametrize("k", [16, 32, 64, 128])
def test_hadamard_constant_is_correctly_rounded(orc, k):
    getcontext().prec = 60
    exact = Decimal(1) / Decimal(k).sqrt()
    c = orc.hadamard_ck(k)
    ulp = Decimal(float(np.spacing(c)))
    assert abs(Decimal(float(c)) - exact) <= ulp / 2
    if k in (16, 64):
        assert float(c) == 1 / math.sqrt(k)


@pytest.mark.parametrize("fmt,k", [(0, 32), (1, 16), (0, 128), (1, 64)])
def test_eq2_norm_identity(orc, fmt, k):
    """||x - H^T Q(Hx)|| == ||Hx - Q(Hx)|| ('Portable FP4 quantization' Eq.(2))."""
    x = _rand_bf16(4, 512, 11)
    q, s, sg = orc.quantize(x, fmt, hadamard_k=k)
    back = orc.dequantize(q, s, sg, fmt, hadamard_k=k).astype(np.float64)
    qhx = orc.dequantize(q, s, sg, fmt, hadamard_k=0).astype(np.float64)
    xf = inputs.bf16_bits_to_f32(x)
    hx = np.stack([orc.fwht(row, k) for row in xf]).astype(np.float64)
    lhs = np.linalg.norm(xf.astype(np.float64) - back)
    rhs = np.linalg.norm(hx - qhx)
    assert abs(lhs - rhs) <= 1e-4 * rhs


def test_rotation_preserves_product(orc):
    rng = np.random.default_rng(4)
    X = rng.standard_normal((6, 256)).astype(np.float32)
    W = rng.standard_normal((5, 256)).astype(np.float32)
    XH = np.stack([orc.fwht(r, 64) for r in X]).astype(np.float64)
    WH = np.stack([orc.fwht(r, 64) for r in W]).astype(np.float64)
    assert np.allclose(XH @ WH.T, X.astype(np.float64) @ W.astype(np.float64).T, atol=1e-4)


# ---------------------------------------------------------------- layout ------
def test_scale_atoms_roundtrip_and_positions(orc):
    rng = np.random.default_rng(2)
    s = rng.integers(1, 255, (200, 10), dtype=np.uint8)
    a = orc.scales_to_atoms(s)
    assert a.size == 256 * 12
    assert np.array_equal(orc.scales_from_atoms(a, 200, 10), s)
    nkb4 = 3
    # row 33, scale column 5 -> atom (0, 1), in-atom (33 % 32)*16 + 1*4 + 1
    assert a[(0 * nkb4 + 1) * 512 + 1 * 16 + 1 * 4 + 1] == s[33, 5]
    # row 130, column 9 -> atom (1, 2), in-atom 2*16 + 0*4 + 1
    assert a[(1 * nkb4 + 2) * 512 + 2 * 16 + 1] == s[130, 9]
    assert np.count_nonzero(a) == s.size  # padding is zero


# ---------------------------------------------------------------- GEMM -------
def test_gemm_reference_equals_numpy(orc):
    rng = np.random.default_rng(0)
    a = rng.standard_normal((7, 96)).astype(np.float32)
    w = rng.standard_normal((9, 96)).astype(np.float32)
    c, b = orc.gemm_ref(a, w)
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert np.allclose(c, ref, rtol=1e-13, atol=1e-12)
    assert np.allclose(b, np.abs(a).astype(np.float64) @ np.abs(w).astype(np.float64).T, rtol=1e-13)
    # not transposed: an asymmetric case must not equal A^T-style products
    assert not np.allclose(c[:7, :7], c[:7, :7].T)


def test_tiny_linear_end_to_end(orc):
    a, w = inputs.tiny_linear()
    qa, sa, _ = orc.quantize(a, 0)
    qw, sw, _ = orc.quantize(w, 0)
    ah = orc.dequantize(qa, sa, 1.0, 0)
    wh = orc.dequantize(qw, sw, 1.0, 0)
    c, b = orc.gemm_ref(ah, wh)
    ref = ah.astype(np.float64) @ wh.astype(np.float64).T
    assert np.allclose(c, ref, rtol=1e-12, atol=1e-12)
    # sanity: 4-bit operands with 1% x20 outliers keep the product within ~20%
    exact = inputs.bf16_bits_to_f32(a).astype(np.float64) @ inputs.bf16_bits_to_f32(w).astype(np.float64).T
    assert np.linalg.norm(c - exact) / np.linalg.norm(exact) < 0.3


# ---------------------------------------------------------------- statistics --
def test_table5_nmse_directional(orc):
    """Directional check against Table 5: NVFP4 < rotated MXFP4 < MXFP4, each
    within a factor 2 of the printed NMSE (the page's generator is unknown)."""
    g = golden("table5_nmse.txt")
    for key, gen in (("act_1pct", inputs.table5_activation), ("w_0.3pct", inputs.table5_weight)):
        want = {m: float(v) for m, v in g[key]}
        xf = gen()
        x = inputs.f32_to_bf16_bits(xf.reshape(1, -1))
        xb = inputs.bf16_bits_to_f32(x)
        got = {}
        for name, fmt, k in (("mxfp4", 0, 0), ("nvfp4", 1, 0), ("rot_mxfp4", 0, 32)):
            q, s, sg = orc.quantize(x, fmt, hadamard_k=k)
            got[name] = orc.nmse(xb, orc.dequantize(q, s, sg, fmt, hadamard_k=k))
        assert got["nvfp4"] < got["rot_mxfp4"] < got["mxfp4"]
        for m in got:  # the INT4 / TransFP4 rows are pinned in test_oracle_transfp4_pins.py
            v = want[m]
            assert v / 2 < got[m] < v * 2, (key, m, got[m], v)


# ---- quantization of fp32 elements (a product quantized for the next layer) ----
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hk,tie", [(0, 0), (32, 0), (0, 1)])
def test_quantize_f32_equals_bf16_path_on_bf16_values(orc, fmt, hk, tie):
    """Widening bf16 to fp32 is exact, so the fp32 entry point must give the
    bf16 one's bytes on every bf16 tensor."""
    x = inputs.quant_sweep(rows=24, cols=1024, seed=17)
    a = orc.quantize(x, fmt, hadamard_k=hk, tie=tie)
    b = orc.quantize_f32(inputs.bf16_bits_to_f32(x), fmt, hadamard_k=hk, tie=tie)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


@pytest.mark.parametrize("tie", [0, 1])
def test_quantize_f32_brute_force_nearest(orc, tie):
    """Blocks whose largest magnitude is exactly 6 get scale 1 (MXFP4 byte 127;
    NVFP4 with s_g = 1: block scale 1.0 = 0x38), so every other element's code
    must be the nearest E2M1 value found by brute force over the grid, ties by
    the rule; the values are fp32 ones a bf16 tensor cannot hold."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    rng = np.random.default_rng(23)
    v = rng.uniform(-6, 6, (8, 64)).astype(np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    v[:, 1:8] = mids                                  # exact midpoints
    v[:, 8:15] = np.nextafter(mids, np.float32(10))   # just above them
    v[:, 15:22] = np.nextafter(mids, np.float32(-10)) # just below them
    v[:, 0] = 6.0
    v[:, 32] = -6.0                                   # second MX block's max, both NV blocks of it too
    v[:, 16] = 6.0                                    # the other NV blocks' max
    v[:, 48] = 6.0

    def nearest(a):
        d = np.abs(grid - abs(float(a)))
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:  # a midpoint
            i = best[-1] if tie == 1 else (best[0] if best[0] % 2 == 0 else best[1])
        else:
            i = best[0]
        return int(i) | (8 if np.signbit(a) else 0)

    want = np.array([[nearest(a) for a in row] for row in v])
    for fmt, gs in ((0, None), (1, 1.0)):
        q, s, _ = orc.quantize_f32(v, fmt, tie=tie, gscale=gs)
        codes = np.zeros_like(want)
        codes[:, 0::2] = q & 0xF
        codes[:, 1::2] = q >> 4
        assert np.array_equal(codes, want), fmt
        assert np.all(s == (127 if fmt == 0 else 0x38))


# ----------------------------------------------------- MXFP4 -> NVFP4 scales ----
def test_mx_to_nv_scales_keep_every_element(orc):
    """Late binding of an MXFP4 weight to the NVFP4 scale form ("Portable FP4
    quantization (TransFP4)" §2.5): the same E2M1 codes dequantize to the same
    values, bit for bit, for weights whose block scales span <= 17 binades."""
    for seed, fmt_rows in ((0, (64, 512)), (1, (37, 1024)), (2, (128, 4096))):
        rows, cols = fmt_rows
        rng = np.random.default_rng(seed)
        w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (rows, cols)).astype(np.float32))
        q, s_mx, _ = orc.quantize(w, orc.MXFP4)
        s_nv, g = orc.mx_scales_to_nv(s_mx)
        assert s_nv.shape == (rows, cols // 16)
        a = orc.dequantize(q, s_mx, 1.0, orc.MXFP4)
        b = orc.dequantize(q, s_nv, g, orc.NVFP4)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_mx_to_nv_scales_closed_form(orc):
    """s_g = 2^(e_max - 8); each 2^e becomes 2^(e - E) in E4M3: normal codes
    (exponent field e - E + 7, mantissa 0), subnormals 2^-7, 2^-8, 2^-9 as
    mantissa 4, 2, 1, and 2^-10 (a tie with 0) and below as 0."""
    e_max = 13
    E = e_max - 8
    es = [e_max, 0, e_max - 14, e_max - 15, e_max - 16, e_max - 17, e_max - 18, e_max - 40]
    want = [0x78, ((0 - E) + 7) << 3, 0x08, 0x04, 0x02, 0x01, 0x00, 0x00]
    s_mx = np.array([[e + 127 for e in es]], np.uint8)
    s_nv, g = orc.mx_scales_to_nv(s_mx)
    assert g == 2.0 ** E
    assert s_nv[0, 0::2].tolist() == want and s_nv[0, 1::2].tolist() == want
    for e, b in zip(es, want):
        if b:
            assert orc.e4m3_decode(b) * g == 2.0 ** e
    # NaN scale, and a tensor of zero blocks (s_g clamped to the smallest normal float)
    s_nv, g = orc.mx_scales_to_nv(np.array([[0xFF, 127]], np.uint8))
    assert s_nv[0, :2].tolist() == [0x7F, 0x7F]
    s_nv, g = orc.mx_scales_to_nv(np.zeros((2, 4), np.uint8))
    assert g == 2.0 ** -126 and (s_nv == 0x30).all()


# ------------------------------------------------------- sparse residual lane ----
def _units_top_zeroed(y):
    """Rotated rows y (fp32): the first largest-magnitude value of every
    32-value unit and its index, and y with those values zeroed."""
    u = y.reshape(y.shape[0], -1, 32)
    idx = np.abs(u).argmax(-1)                       # first of equal maxima
    top = np.take_along_axis(u, idx[..., None], -1)[..., 0]
    z = u.copy()
    np.put_along_axis(z, idx[..., None], 0.0, -1)
    return top, idx, z.reshape(y.shape)


def _rotate_rows(orc, x_bf16, hk):
    y = inputs.bf16_bits_to_f32(x_bf16).astype(np.float32).copy()
    if hk:
        for r in range(y.shape[0]):
            y[r] = orc.fwht(y[r], hk)
    return y


@pytest.mark.parametrize("fmt,hk,gscale", [(0, 0, None), (0, 32, None), (1, 0, None), (1, 32, None), (1, 16, 0.01)])
def test_residual_lane_fp4_stream_is_the_plain_quantizer(orc, fmt, hk, gscale):
    """TransFP4 Eq.(3): Q_f(Hx - P_r Hx) is the ordinary quantizer applied to
    the rotated values with each unit's largest one zeroed (also for the
    NVFP4 tensor scale, taken from that stream); the residual word holds the
    bf16 rounding (torch's) of that value and its index."""
    import torch
    x = inputs.f32_to_bf16_bits(inputs.table5_activation(64 * 512, seed=3).reshape(64, 512))
    q, s, g, res = orc.quantize_residual(x, fmt, hadamard_k=hk, gscale=gscale)
    y = _rotate_rows(orc, x, hk)
    top, idx, z = _units_top_zeroed(y)
    q2, s2, g2 = orc.quantize_f32(z, fmt, gscale=gscale)
    assert np.array_equal(q, q2) and np.array_equal(s, s2) and g == g2
    want_bits = torch.from_numpy(top.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(res & 0xFFFF, want_bits.astype(np.uint32))
    assert np.array_equal(res >> 16, idx.astype(np.uint32))


def test_residual_lane_one_value_units_exact(orc):
    """Units holding one nonzero bf16 value: the FP4 stream is all zero and
    Eq.(3) returns the input exactly."""
    rng = np.random.default_rng(9)
    v = np.zeros((8, 256), np.float32)
    for r in range(8):
        for u in range(8):
            v[r, u * 32 + rng.integers(0, 32)] = rng.laplace(0, 3)
    x = inputs.f32_to_bf16_bits(v)
    for fmt in (0, 1):
        q, s, g, res = orc.quantize_residual(x, fmt)
        assert not q.any()
        xh = orc.dequantize_residual(q, s, g, res, fmt)
        assert np.array_equal(xh, inputs.bf16_bits_to_f32(x))


@pytest.mark.parametrize("fmt", [0, 1])
def test_residual_lane_lowers_the_error(orc, fmt):
    """On the Table 4 activation tensor (1 % outliers) the residual lane lowers
    the NMSE of the same quantizer without it, with H = I and with H_32.
    (Measured: MXFP4 0.0281 -> 0.0066 and 0.0120 -> 0.0102; NVFP4 0.0083 ->
    0.0033 and 0.0102 -> 0.0091.)"""
    xf = inputs.table5_activation()
    x = inputs.f32_to_bf16_bits(xf.reshape(-1, 1024))
    xs = inputs.bf16_bits_to_f32(x)
    for hk in (0, 32):
        q, s, g = orc.quantize(x, fmt, hadamard_k=hk)
        base = orc.nmse(xs, orc.dequantize(q, s, g, fmt, hadamard_k=hk))
        q, s, g, res = orc.quantize_residual(x, fmt, hadamard_k=hk)
        lane = orc.nmse(xs, orc.dequantize_residual(q, s, g, res, fmt, hadamard_k=hk))
        assert lane < base, (hk, lane, base)
    if fmt == 0:
        assert lane < 0.5 * orc.nmse(xs, orc.dequantize(*orc.quantize(x, fmt), fmt))
