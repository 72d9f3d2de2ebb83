"""GPU parity of the GEMM paths when K is a multiple of 32 but not of 256
("Portable FP4 quantization (TransFP4)" Table 3: the GEMM's K alignment is
32).  The kernels step K by 256; the last step reads zeros past K (TMA fill)
and the zero padding scales of the tile layout, so the result is the oracle's
product over the K real elements: bit-exact with unit scales, within
1e-5 * sum_k |a||w| otherwise.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import to_dev_bf16, to_np

pytestmark = pytest.mark.gpu

KS = [32, 96, 288, 800, 4128]


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
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(), torch.from_numpy(orc.scales_to_atoms(s_logical)).cuda(),
            torch.tensor([g], dtype=torch.float32, device="cuda"))


def reference(orc, qa, sa, ga, qw, sw, gw, fmt):
    return orc.gemm_ref(orc.dequantize(qa, sa, ga, fmt), orc.dequantize(qw, sw, gw, fmt))


def assert_close(c, ref, bound):
    err = np.abs(np.asarray(c, np.float64) - ref)
    bad = np.argwhere(err > 1e-5 * bound)
    assert bad.size == 0, f"{bad.shape[0]} out of tolerance, first {bad[:3].tolist()}"


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("K", KS)
@pytest.mark.parametrize("M,N", [(1, 1000), (16, 4096), (130, 300), (256, 512)])
def test_gemm_k_tail_unit_scales_exact(fp4, orc, fmt, K, M, N):
    """Decode (M <= 16: whole tiles, cluster and global splits) and the tiled
    kernel (one and two CTAs per tile)."""
    import torch
    rng = np.random.default_rng(M + N + K + fmt)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    B = 32 if fmt == 0 else 16
    unit = 127 if fmt == 0 else 0x38
    sa = np.full((M, K // B), unit, np.uint8)
    sw = np.full((N, K // B), unit, np.uint8)
    c = fp4.gemm(upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, fmt, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    ref, _ = reference(orc, qa, sa, 1.0, qw, sw, 1.0, fmt)
    assert np.array_equal(to_np(c).astype(np.float64), ref)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("K", [96, 800, 4128])
@pytest.mark.parametrize("M,N", [(4, 14336), (200, 520)])
def test_gemm_k_tail_random(fp4, orc, fmt, K, M, N):
    import torch
    rng = np.random.default_rng(3 * M + N + K)
    a = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qa, sa, ga = orc.quantize(a, fmt)
    qw, sw, gw = orc.quantize(w, fmt)
    c = fp4.gemm(upload(orc, qa, sa, ga), upload(orc, qw, sw, gw), M, N, K, fmt, out_dtype=0)
    torch.cuda.synchronize()
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(to_np(c), ref, bound)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("K,hk", [(96, 32), (288, 0), (4128, 32)])
@pytest.mark.parametrize("M", [1, 5, 16, 200])
def test_linear_k_tail(fp4, orc, fmt, K, hk, M):
    """fp4_linear: online activation quantization (one-cluster quantizer for
    M <= 16, streaming quantizer above) and the product, against the oracle.
    The workspace starts as 0xFF bytes, NaN as scales of either format: the
    activation quantizer must write the padding scale columns the last K step
    reads."""
    import torch
    N = 1000
    rng = np.random.default_rng(M + K + hk + fmt)
    x = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qw, sw, gw = orc.quantize(w, fmt, hadamard_k=hk)
    ws = torch.full((fp4.linear_workspace_size(M, N, K, fmt),), 0xFF, dtype=torch.uint8, device="cuda")
    c = fp4.linear(to_dev_bf16(x), upload(orc, qw, sw, gw), fmt, hadamard_k=hk, out_dtype=0, workspace=ws)
    torch.cuda.synchronize()
    fp4.check_device_status()
    qa, sa, ga = orc.quantize(x, fmt, hadamard_k=hk)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(to_np(c), ref, bound)


@pytest.mark.parametrize("fmt,out_fmt", [(0, 0), (1, 1)])
def test_gemm_quantized_k_tail(fp4, orc, fmt, out_fmt):
    """The quantizing epilogue over a K tail, unit scales: exact."""
    import torch
    M, N, K = 256, 384, 288
    rng = np.random.default_rng(7 + fmt)
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    B = 32 if fmt == 0 else 16
    unit = 127 if fmt == 0 else 0x38
    sa, sw = np.full((M, K // B), unit, np.uint8), np.full((N, K // B), unit, np.uint8)
    ref, _ = reference(orc, qa, sa, 1.0, qw, sw, 1.0, fmt)
    gC = float(np.float32(np.abs(ref).max() / 2688)) if out_fmt == 1 else None
    gs = None if gC is None else torch.tensor([gC], dtype=torch.float32, device="cuda")
    Cq, Cs, _ = fp4.gemm_quantized(upload(orc, qa, sa, 1.0), upload(orc, qw, sw, 1.0), M, N, K, fmt, out_fmt,
                                   gscale=gs)
    torch.cuda.synchronize()
    eq, es, _ = orc.quantize_f32(ref.astype(np.float32), out_fmt, gscale=gC)
    assert np.array_equal(to_np(Cq), eq)
    assert np.array_equal(to_np(Cs), orc.scales_to_atoms(es))
