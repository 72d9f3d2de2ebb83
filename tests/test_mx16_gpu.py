"""GPU parity of MXFP4 on 16-element blocks (FP4_MXFP4_16: E2M1 elements,
one E8M0 scale per 16 consecutive K elements; "Portable FP4 quantization
(TransFP4)" §1.1 Eq.(1) with block size G = 16, the scale encoding of "4.5
FP8 and NVFP4/MXFP4" §3.3's MXFP4).

Quantization: packed nibbles and scale bytes (tile layout, padding included)
bit-exact against the oracle; dequantized fp32 values bit-exact, bf16 their
RNE rounding.  Product: the 16-element block-scaled MMA with E8M0 scales,
exact with unit scales, within 1e-5 * sum_k |a||w| of the oracle's fp64
product otherwise, as is the NVFP4 product of the same elements whose E4M3
block scales hold the same powers of two.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import bf16_tensor_bits, to_dev_bf16, to_np

pytestmark = pytest.mark.gpu

MX16 = 2


@pytest.fixture(scope="module")
def fp4():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_microscaling_quantization_b200 import build
    build.build()
    import fp4_microscaling_quantization_b200 as m
    return m


def check_quantize(fp4, orc, x, hk=0, tie=0, rule=0, search=0):
    import torch
    q, s, g = fp4.quantize(to_dev_bf16(x), MX16, hadamard_k=hk, round=tie, mx_scale_rule=rule,
                           scale_search=search)
    torch.cuda.synchronize()
    oq, os_, og = orc.quantize(x, orc.MXFP4_16, hadamard_k=hk, tie=tie, mx_rule=rule, search=search)
    bad = np.argwhere(to_np(q) != oq)
    assert bad.size == 0, f"nibbles differ at {bad[:4].tolist()}"
    sbad = np.flatnonzero(to_np(s) != orc.scales_to_atoms(os_))
    assert sbad.size == 0, f"scales differ at {sbad[:4].tolist()}"
    return q, s, g, (oq, os_, og)


def edge_tensor():
    rows = [np.zeros(64, np.float32), -np.zeros(64, np.float32)]
    rows.append(np.array([(i + 1) * 2.0 ** -133 for i in range(64)], np.float32))  # bf16 subnormals
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 8, np.float32)
    rows.append(ties * np.where(np.arange(64) % 3 == 0, -1, 1))
    rows.append(ties * 2.0 ** 20)
    r = np.full(64, 1e-3, np.float32)
    r[5], r[40] = 1e4, -3e5
    rows.append(r)
    rows.append(np.linspace(-3e38, 3e38, 64).astype(np.float32))
    return inputs.f32_to_bf16_bits(np.stack(rows))


@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (130, 512), (257, 1024), (37, 3104), (5, 32736)])
def test_quantize_parity_shapes(fp4, orc, shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    v = rng.laplace(0, 1, shape).astype(np.float32)
    v[rng.random(shape) < 0.01] *= 20
    check_quantize(fp4, orc, inputs.f32_to_bf16_bits(v))


@pytest.mark.parametrize("hk", [16, 32, 64, 128])
def test_quantize_parity_rotated(fp4, orc, hk):
    check_quantize(fp4, orc, inputs.rotate_acts(rows=136, cols=1024, seed=hk), hk=hk)


@pytest.mark.parametrize("tie,rule", [(1, 0), (0, 1), (1, 1)])
def test_quantize_parity_modes(fp4, orc, tie, rule):
    x = inputs.quant_sweep(rows=40, cols=2048, seed=9)
    check_quantize(fp4, orc, x, hk=32, tie=tie, rule=rule)
    check_quantize(fp4, orc, x, tie=tie, rule=rule)


@pytest.mark.parametrize("tie", [0, 1])
def test_quantize_edge_cases(fp4, orc, tie):
    x = edge_tensor()
    check_quantize(fp4, orc, x, tie=tie)
    check_quantize(fp4, orc, x[:6], tie=tie, hk=64)


@pytest.mark.parametrize("hk,tie", [(0, 0), (0, 1), (32, 0), (128, 1)])
def test_quantize_mse_search(fp4, orc, hk, tie):
    check_quantize(fp4, orc, inputs.rotate_acts(rows=64, cols=1024, seed=3 + hk), hk=hk, tie=tie, search=1)


@pytest.mark.parametrize("hk", [0, 128])
def test_full_size_rotate(fp4, orc, hk):
    """8192 x 4096 activations with outlier channels."""
    check_quantize(fp4, orc, inputs.rotate_acts(), hk=hk)


@pytest.mark.parametrize("hk", [0, 32, 128])
@pytest.mark.parametrize("bf16", [0, 1])
def test_dequantize_parity(fp4, orc, hk, bf16):
    import torch
    x = inputs.rotate_acts(rows=130, cols=512, seed=5)
    q, s, g, (oq, os_, og) = check_quantize(fp4, orc, x, hk=hk)
    out = fp4.dequantize(q, s, g, MX16, hadamard_k=hk, out_dtype=bf16)
    torch.cuda.synchronize()
    ref = orc.dequantize(oq, os_, og, orc.MXFP4_16, hadamard_k=hk)
    if bf16:
        assert np.array_equal(bf16_tensor_bits(out), inputs.f32_to_bf16_bits(ref))
    else:
        assert np.array_equal(to_np(out).view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("hk", [0, 32])
def test_residual_lane(fp4, orc, hk):
    import torch
    x = inputs.rotate_acts(rows=70, cols=1024, seed=11)
    q, s, g, res = fp4.quantize_residual(to_dev_bf16(x), MX16, hadamard_k=hk)
    torch.cuda.synchronize()
    oq, os_, og, ores = orc.quantize_residual(x, orc.MXFP4_16, hadamard_k=hk)
    assert np.array_equal(to_np(q), oq)
    assert np.array_equal(to_np(s), orc.scales_to_atoms(os_))
    assert np.array_equal(to_np(res).view(np.uint32), ores)
    out = fp4.dequantize_residual(q, s, g, res, MX16, hadamard_k=hk)
    torch.cuda.synchronize()
    ref = orc.dequantize_residual(oq, os_, og, ores, orc.MXFP4_16, hadamard_k=hk)
    assert np.array_equal(to_np(out).view(np.uint32), ref.view(np.uint32))


def test_block_16_spelling(fp4, orc):
    """fmt = FP4_MXFP4 with block = 16 is the same format as FP4_MXFP4_16."""
    import torch
    from fp4_microscaling_quantization_b200 import _lib
    x = inputs.quant_sweep(rows=20, cols=512, seed=2)
    q1, s1, _ = fp4.quantize(to_dev_bf16(x), MX16)
    q2, s2 = torch.empty_like(q1), torch.empty_like(s1)
    xd = to_dev_bf16(x)
    _lib.check("fp4_quantize", _lib.lib().fp4_quantize(
        xd.data_ptr(), 20, 512, 512, 0, 16, 0, None, q2.data_ptr(), s2.data_ptr(), None,
        torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1, s2)


# ----------------------------------------------------------------- product ---
def upload(orc, q, s_logical):
    import torch
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(), torch.from_numpy(orc.scales_to_atoms(s_logical)).cuda(),
            torch.ones((1,), dtype=torch.float32, device="cuda"))


def assert_close(c, ref, bound):
    err = np.abs(np.asarray(c, np.float64) - ref)
    bad = np.argwhere(err > 1e-5 * bound)
    assert bad.size == 0, f"{bad.shape[0]} out of tolerance, first {bad[:3].tolist()}"


GEMM_SHAPES = [(1, 1000, 1024), (4, 4096, 4128), (16, 14336, 512), (130, 300, 512), (256, 512, 800),
               (300, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_unit_scales_exact(fp4, orc, M, N, K):
    """Scale byte 127 (2^0) on every 16-block: the product of the E2M1 codes,
    exact in fp32 at these K."""
    import torch
    rng = np.random.default_rng(M + N + K)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = np.full((M, K // 16), 127, np.uint8)
    sw = np.full((N, K // 16), 127, np.uint8)
    c = fp4.gemm(upload(orc, qa, sa), upload(orc, qw, sw), M, N, K, MX16, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, orc.MXFP4_16), orc.dequantize(qw, sw, 1.0, orc.MXFP4_16))
    assert np.array_equal(to_np(c).astype(np.float64), ref)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_random(fp4, orc, M, N, K):
    import torch
    rng = np.random.default_rng(3 * M + N + K)
    a = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qa, sa, _ = orc.quantize(a, orc.MXFP4_16)
    qw, sw, _ = orc.quantize(w, orc.MXFP4_16)
    c = fp4.gemm(upload(orc, qa, sa), upload(orc, qw, sw), M, N, K, MX16, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    ref, bound = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, orc.MXFP4_16), orc.dequantize(qw, sw, 1.0, orc.MXFP4_16))
    assert_close(to_np(c), ref, bound)


@pytest.mark.parametrize("M,N,K", [(4, 1000, 1024), (200, 768, 2048)])
def test_gemm_agrees_with_nvfp4_on_the_same_scales(fp4, orc, M, N, K):
    """E8M0 scales 2^e with e in [-9, 8] are also E4M3 values (code
    8 (e + 7) for e >= -6, the subnormals 2^-7 .. 2^-9 below).  With s_g = 1
    the NVFP4 product of the same elements is the same sum of the same
    products, so both kernels' results lie within the tolerance of the
    oracle's: the MMA reads the MXFP4_16 scale bytes as E8M0 (read as E4M3,
    bytes near 127 would mean values near 2^8 instead of 2^0)."""
    import torch
    rng = np.random.default_rng(M + K)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ea = rng.integers(-9, 9, (M, K // 16))
    ew = rng.integers(-9, 9, (N, K // 16))

    def e4m3(e):
        return np.where(e >= -6, 8 * (e + 7), 1 << (e + 9)).astype(np.uint8)

    mx = fp4.gemm(upload(orc, qa, (ea + 127).astype(np.uint8)), upload(orc, qw, (ew + 127).astype(np.uint8)),
                  M, N, K, MX16, out_dtype=0)
    nv = fp4.gemm(upload(orc, qa, e4m3(ea)), upload(orc, qw, e4m3(ew)), M, N, K, fp4.FP4_NVFP4, out_dtype=0)
    torch.cuda.synchronize()
    assert orc.e4m3_decode(int(e4m3(np.array(-9)))) == 2.0 ** -9 and orc.e4m3_decode(int(e4m3(np.array(8)))) == 256.0
    sa = (ea + 127).astype(np.uint8)
    sw = (ew + 127).astype(np.uint8)
    ref, bound = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, orc.MXFP4_16), orc.dequantize(qw, sw, 1.0, orc.MXFP4_16))
    ref_nv, _ = orc.gemm_ref(orc.dequantize(qa, e4m3(ea), 1.0, orc.NVFP4), orc.dequantize(qw, e4m3(ew), 1.0, orc.NVFP4))
    assert np.array_equal(ref, ref_nv)  # the same operands, as the oracle dequantizes them
    assert_close(to_np(mx), ref, bound)
    assert_close(to_np(nv), ref, bound)


@pytest.mark.parametrize("M", [1, 5, 16, 200])
@pytest.mark.parametrize("K,hk", [(1024, 0), (4096, 32), (800, 32)])
def test_linear(fp4, orc, M, K, hk):
    """fp4_linear: activations quantized online to MXFP4_16 (the one-cluster
    quantizer for M <= 16, the streaming one above) and the product."""
    import torch
    N = 1000
    rng = np.random.default_rng(M + K + hk)
    x = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qw, sw, _ = orc.quantize(w, orc.MXFP4_16, hadamard_k=hk)
    ws = torch.full((fp4.linear_workspace_size(M, N, K, MX16),), 0xFF, dtype=torch.uint8, device="cuda")
    c = fp4.linear(to_dev_bf16(x), upload(orc, qw, sw), MX16, hadamard_k=hk, out_dtype=0, workspace=ws)
    torch.cuda.synchronize()
    fp4.check_device_status()
    qa, sa, _ = orc.quantize(x, orc.MXFP4_16, hadamard_k=hk)
    ref, bound = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, orc.MXFP4_16), orc.dequantize(qw, sw, 1.0, orc.MXFP4_16))
    assert_close(to_np(c), ref, bound)


@pytest.mark.parametrize("out_fmt", [0, 1])
def test_gemm_quantized_unit_scales(fp4, orc, out_fmt):
    """MXFP4_16 operands, C quantized in the epilogue to MXFP4 / NVFP4: exact
    with unit scales."""
    import torch
    M, N, K = 256, 384, 544
    rng = np.random.default_rng(40 + out_fmt)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa, sw = np.full((M, K // 16), 127, np.uint8), np.full((N, K // 16), 127, np.uint8)
    ref, _ = orc.gemm_ref(orc.dequantize(qa, sa, 1.0, orc.MXFP4_16), orc.dequantize(qw, sw, 1.0, orc.MXFP4_16))
    gC = float(np.float32(np.abs(ref).max() / 2688)) if out_fmt == 1 else None
    gs = None if gC is None else torch.tensor([gC], dtype=torch.float32, device="cuda")
    Cq, Cs, _ = fp4.gemm_quantized(upload(orc, qa, sa), upload(orc, qw, sw), M, N, K, MX16, out_fmt, gscale=gs)
    torch.cuda.synchronize()
    eq, es, _ = orc.quantize_f32(ref.astype(np.float32), out_fmt, gscale=gC)
    assert np.array_equal(to_np(Cq), eq)
    assert np.array_equal(to_np(Cs), orc.scales_to_atoms(es))
