"""GPU parity of fp4_gemm_quantized: the prefill GEMM whose epilogue quantizes
C = alpha * A W^T along N for the next layer ("FP4 quantization analysis:
MXFP4 vs NVFP4" §3.3, the QuTLASS fused epilogue; TransFP4 §1.1 Eq.(1) for the
encoding of each 32-element unit).

The expected bytes are the oracle's quantization of the oracle's product.
Where every partial sum of the product is exact in FP32 (E2M1 codes times
power-of-two scales, small K), C is bit-exact on the GPU and so must be every
element code and scale byte.  For general inputs the FP32 accumulation may
differ from the fp64 product by up to 1e-5 * sum_k |a||w|, which can move a
value across a rounding midpoint: there the scale bytes may differ by one
step and the element codes by one position, in a small fraction of places.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import to_dev_bf16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp4():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_microscaling_quantization_b200 import build
    build.build()
    import fp4_microscaling_quantization_b200 as m
    return m


def upload(orc, q, s_logical, g):
    import torch
    qd = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    sd = torch.from_numpy(orc.scales_to_atoms(s_logical)).cuda()
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    return qd, sd, gd


def run(fp4, A, W, M, N, K, fmt, out_fmt, gC=None, **kw):
    """fp4_gemm_quantized into sentinel-filled buffers; checks that nothing
    past the M rows of elements is written and returns the host copies."""
    import torch
    qb, sb = fp4.quantize_sizes(M, N, out_fmt)
    q_full = torch.full((M + 1, N // 2), 0xA5, dtype=torch.uint8, device="cuda")
    Cs = torch.full((sb,), 0xEE, dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    gs = None if gC is None else torch.tensor([gC], dtype=torch.float32, device="cuda")
    fp4.gemm_quantized(A, W, M, N, K, fmt, out_fmt, gscale=gs, out=(q_full[:M], Cs, g), **kw)
    torch.cuda.synchronize()
    fp4.check_device_status()
    qf = to_np(q_full)
    assert (qf[M] == 0xA5).all(), "elements written past row M"
    return qf[:M], to_np(Cs)


def signed_index(q):
    """Packed nibbles -> signed position on the E2M1 grid (-7..7)."""
    lo, hi = q & 15, q >> 4
    c = np.stack([lo, hi], -1).reshape(q.shape[0], -1).astype(np.int32)
    return np.where(c & 8, -(c & 7), c & 7)


def block_of(fmt):
    return 32 if fmt == 0 else 16


def assert_exact(orc, q, s_atoms, ref, M, N, out_fmt, gC=None, **kw):
    c32 = ref.astype(np.float32)
    assert np.array_equal(c32.astype(np.float64), ref), "test product is not exact in FP32"
    eq, es, _ = orc.quantize_f32(c32, out_fmt, gscale=gC, **kw)
    assert np.array_equal(q, eq), f"{np.count_nonzero(q != eq)} element bytes differ"
    ea = orc.scales_to_atoms(es)
    assert np.array_equal(s_atoms, ea), f"{np.count_nonzero(s_atoms != ea)} scale bytes differ"


def assert_within_one_step(orc, q, s_atoms, ref, M, N, out_fmt, gC=None, frac=1e-3, rows=None):
    """Scales within one step of the oracle's quantization of fp32(ref) and
    equal almost everywhere; element codes, in blocks with equal scales,
    within one grid position and equal almost everywhere.  `rows` selects
    the rows of the GPU output that `ref` holds."""
    nkb = N // block_of(out_fmt)
    Mpad = (M + 127) // 128 * 128
    eq, es, _ = orc.quantize_f32(ref.astype(np.float32), out_fmt, gscale=gC)
    s_all = orc.scales_from_atoms(s_atoms, Mpad, nkb)
    assert (s_all[M:] == 0).all(), "padding rows of the scale layout not zeroed"
    gs = s_all[:M] if rows is None else s_all[rows]
    gq = q if rows is None else q[rows]
    ds = np.abs(gs.astype(np.int32) - es.astype(np.int32))
    assert ds.max(initial=0) <= 1 and np.count_nonzero(ds) <= frac * ds.size, (ds.max(), np.count_nonzero(ds))
    same = np.repeat(ds == 0, block_of(out_fmt), axis=1)
    dq = np.abs(signed_index(gq) - signed_index(eq))[same]
    assert dq.max(initial=0) <= 1 and np.count_nonzero(dq) <= frac * dq.size, (dq.max(), np.count_nonzero(dq))


def rand_q(rng, rows, K):
    return rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)


def unit_scales(fmt, rows, K):
    return np.full((rows, K // block_of(fmt)), 127 if fmt == 0 else 0x38, np.uint8)


def pow2_scales(rng, fmt, rows, K):
    """Scales 2^-1, 2^0, 2^1: E8M0 126..128, E4M3 0x30, 0x38, 0x40."""
    pick = rng.integers(0, 3, (rows, K // block_of(fmt)))
    return (np.array([126, 127, 128], np.uint8) if fmt == 0 else np.array([0x30, 0x38, 0x40], np.uint8))[pick]


def nv_gscale(ref):
    amax = float(np.abs(ref).max())
    return float(np.float32(amax / 2688.0)) if amax > 0 else 1.0


SHAPES = [(256, 256, 512), (300, 384, 256), (64, 128, 1024), (130, 512, 256), (17, 640, 256)]


@pytest.mark.parametrize("fmt,out_fmt", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("shape", SHAPES)
def test_unit_scale_exact(fp4, orc, fmt, out_fmt, shape):
    """Unit operand scales: C is exact, so every byte must match the oracle;
    covers one and two 128-row tiles per CTA, ragged M (zeroed padding rows
    of the scale layout), N = 128 mod 256 and the smallest tiled M."""
    M, N, K = shape
    rng = np.random.default_rng(M * 7 + N + K + fmt * 3 + out_fmt)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = unit_scales(fmt, M, K), unit_scales(fmt, N, K)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, fmt), orc.dequantize(qw, sw, 1.0, fmt))
    gC = nv_gscale(ref) if out_fmt == 1 else None
    q, s = run(fp4, upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, fmt, out_fmt, gC)
    assert_exact(orc, q, s, ref, M, N, out_fmt, gC)


@pytest.mark.parametrize("fmt,out_fmt", [(0, 0), (1, 1), (1, 0)])
def test_pow2_scales_and_tensor_scales_exact(fp4, orc, fmt, out_fmt):
    """Block scales 2^-1..2^1 and, for NVFP4 operands, tensor scales 1/2 and
    1/4 (alpha = 1/8): still exact in FP32, so still bit-exact."""
    M, N, K = 256, 384, 512
    rng = np.random.default_rng(31 + fmt + out_fmt)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = pow2_scales(rng, fmt, M, K), pow2_scales(rng, fmt, N, K)
    ga, gw = (0.5, 0.25) if fmt == 1 else (1.0, 1.0)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, ga, fmt), orc.dequantize(qw, sw, gw, fmt))
    gC = nv_gscale(ref) if out_fmt == 1 else None
    q, s = run(fp4, upload(orc, qa, sa, ga), upload(orc, qw, sw, gw), M, N, K, fmt, out_fmt, gC)
    assert_exact(orc, q, s, ref, M, N, out_fmt, gC)


@pytest.mark.parametrize("out_fmt,round,rule", [(0, 1, 0), (0, 0, 1), (0, 1, 1), (1, 1, 0)])
def test_rounding_options_exact(fp4, orc, out_fmt, round, rule):
    """Products of E2M1 codes land on the element grid's midpoints often, so
    ties-away against ties-even and the floor scale rule are visible."""
    M, N, K = 128, 256, 256
    rng = np.random.default_rng(41 + out_fmt * 4 + round * 2 + rule)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = unit_scales(0, M, K), unit_scales(0, N, K)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, 0), orc.dequantize(qw, sw, 1.0, 0))
    gC = nv_gscale(ref) if out_fmt == 1 else None
    q, s = run(fp4, upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, 0, out_fmt, gC,
               round=round, mx_scale_rule=rule)
    assert_exact(orc, q, s, ref, M, N, out_fmt, gC, tie=round, mx_rule=rule)
    if out_fmt == 0:
        # MXFP4 scales are powers of two, so midpoints are common and both options show
        q0, s0 = run(fp4, upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, 0, out_fmt, gC)
        assert not (np.array_equal(q, q0) and np.array_equal(s, s0)), "the option changed nothing here"


def test_given_tensor_scale_saturates(fp4, orc):
    """NVFP4 output with a given s_g 16x too small: block scales clamp at the
    E4M3 maximum and elements at +-6, as the oracle does."""
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(51)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = unit_scales(1, M, K), unit_scales(1, N, K)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, 1), orc.dequantize(qw, sw, 1.0, 1))
    gC = float(np.float32(nv_gscale(ref) / 16))
    q, s = run(fp4, upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, 1, 1, gC)
    assert_exact(orc, q, s, ref, M, N, 1, gC)
    assert (orc.scales_from_atoms(s, M, N // 16) == 0x7E).any()


def test_output_feeds_the_next_gemm(fp4, orc):
    """C1 quantized in the epilogue is the next GEMM's activation operand, in
    the layout it reads: C2 = Q(C1) W2^T equals the oracle's chain exactly."""
    import torch
    M, N1, K1, N2 = 256, 512, 256, 256
    rng = np.random.default_rng(61)
    qa, qw1 = rand_q(rng, M, K1), rand_q(rng, N1, K1)
    qw2 = rand_q(rng, N2, N1)
    sa, sw1, sw2 = unit_scales(0, M, K1), unit_scales(0, N1, K1), unit_scales(0, N2, N1)
    W2 = upload(orc, qw2, sw2, 1.0)
    Cq, Cs, gC = fp4.gemm_quantized(upload(orc, qa, sa, 1.0), upload(orc, qw1, sw1, 1.0), M, N1, K1, 0, 0)
    c2 = to_np(fp4.gemm((Cq, Cs, gC), W2, M, N2, N1, 0, out_dtype=0))
    torch.cuda.synchronize()
    fp4.check_device_status()
    c1, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, 0), orc.dequantize(qw1, sw1, 1.0, 0))
    q1, s1, _ = orc.quantize_f32(c1.astype(np.float32), 0)
    ref2, bound = orc.gemm_ref(orc.dequantize(q1, s1, 1.0, 0), orc.dequantize(qw2, sw2, 1.0, 0))
    assert np.all(np.abs(c2.astype(np.float64) - ref2) <= 1e-5 * bound)


@pytest.mark.parametrize("fmt,out_fmt", [(0, 0), (1, 1), (0, 1)])
@pytest.mark.parametrize("shape", [(200, 512, 1024), (384, 1280, 2048)])
def test_general_inputs_within_one_step(fp4, orc, fmt, out_fmt, shape):
    """Laplace activations with outliers and Laplace weights, quantized by
    the oracle with computed scales: the FP32 product may differ from the
    fp64 one by rounding, so the codes are compared up to one step."""
    M, N, K = shape
    rng = np.random.default_rng(M + N * 3 + K + fmt + 5 * out_fmt)
    va = rng.laplace(0, 1, (M, K)).astype(np.float32)
    va[rng.random((M, K)) < 0.01] *= 20
    vw = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    qa, sa, ga = orc.quantize(inputs.f32_to_bf16_bits(va), fmt)
    qw, sw, gw = orc.quantize(inputs.f32_to_bf16_bits(vw), fmt)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, ga, fmt), orc.dequantize(qw, sw, gw, fmt))
    gC = nv_gscale(ref) if out_fmt == 1 else None
    q, s = run(fp4, upload(orc, qa, sa, ga), upload(orc, qw, sw, gw), M, N, K, fmt, out_fmt, gC)
    assert_within_one_step(orc, q, s, ref, M, N, out_fmt, gC)


@pytest.mark.parametrize("fmt", [0, 1])
def test_full_size_prefill_sampled(fp4, orc, fmt):
    """8192 x 8192 activations times a 28672 x 8192 weight, quantized output
    in the input's format; 8 whole sampled rows (every N unit) against the
    oracle, with the padding-free scale layout checked everywhere."""
    import torch
    M, N, K = 8192, 28672, 8192
    a, w = inputs.prefill_linear()
    A = fp4.quantize(to_dev_bf16(a), fmt)
    W = fp4.quantize(to_dev_bf16(w), fmt)
    del a, w
    rng = np.random.default_rng(2)
    rows = np.sort(np.concatenate([rng.choice(M - 1, 7, replace=False), [M - 1]]))
    nkb = K // block_of(fmt)

    def deq(T, idx, nrows):
        q = to_np(T[0])[idx]
        s_log = orc.scales_from_atoms(to_np(T[1]), nrows, nkb)[idx]
        return orc.dequantize(q, s_log, float(to_np(T[2])[0]), fmt)

    ref, _ = orc.gemm_ref(deq(A, rows, M), deq(W, np.arange(N), N))
    gC = nv_gscale(ref) * 2 if fmt == 1 else None
    q, s = run(fp4, A, W, M, N, K, fmt, fmt, gC)
    assert_within_one_step(orc, q, s, ref, M, N, fmt, gC, rows=rows)
    del A, W
    torch.cuda.empty_cache()
