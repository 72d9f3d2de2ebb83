"""GPU parity of the MXFP4 -> NVFP4 scale repacking (fp4_mx_to_nv_scales,
"Portable FP4 quantization (TransFP4)" §2.5, §3.4) and of the mixed product
it enables: NVFP4 activations (quantized online) against MXFP4 weights, the
literal reading of the decode workload.  Repacked scale bytes and s_g are
bit-exact against the oracle; the product is within the GEMM tolerance of
the oracle's product of the NVFP4-dequantized activations and the
MXFP4-dequantized weights.
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
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(), torch.from_numpy(orc.scales_to_atoms(s_logical)).cuda(),
            torch.tensor([g], dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 288), (130, 512), (300, 4128), (4096, 1024)])
def test_repacked_scales_match_oracle(fp4, orc, rows, cols):
    import torch
    rng = np.random.default_rng(rows + cols)
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (rows, cols)).astype(np.float32))
    q, s_mx, _ = orc.quantize(w, orc.MXFP4)
    W = upload(orc, q, s_mx, 1.0)
    q_d, s_nv, g = fp4.mx_to_nv(W)
    torch.cuda.synchronize()
    want_s, want_g = orc.mx_scales_to_nv(s_mx)
    assert np.float32(to_np(g)[0]) == np.float32(want_g)
    assert np.array_equal(to_np(s_nv), orc.scales_to_atoms(want_s))
    # the repacked tensor dequantizes to the MXFP4 values on the GPU too
    a = fp4.dequantize(W[0], W[1], W[2], fp4.FP4_MXFP4, out_dtype=0)
    b = fp4.dequantize(q_d, s_nv, g, fp4.FP4_NVFP4, out_dtype=0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_repacked_scales_wide_range(fp4, orc):
    """Block exponents spread over 40 binades, NaN and zero blocks: the
    small ones round to E4M3 subnormals or 0 exactly as in the oracle."""
    import torch
    rows, cols = 128, 1024
    rng = np.random.default_rng(5)
    s_mx = rng.integers(90, 131, (rows, cols // 32)).astype(np.uint8)
    s_mx[3, 5] = 0xFF
    s_mx[7, :] = 0
    q = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    W = upload(orc, q, s_mx, 1.0)
    _, s_nv, g = fp4.mx_to_nv(W)
    torch.cuda.synchronize()
    want_s, want_g = orc.mx_scales_to_nv(s_mx)
    assert np.float32(to_np(g)[0]) == np.float32(want_g)
    assert np.array_equal(to_np(s_nv), orc.scales_to_atoms(want_s))


@pytest.mark.parametrize("M", [1, 4, 16, 200])
@pytest.mark.parametrize("N,K", [(1000, 1024), (4096, 4128)])
def test_nvfp4_activations_mxfp4_weights(fp4, orc, M, N, K):
    """fp4_linear with fmt = NVFP4 on an MXFP4 weight bound to the NVFP4 form:
    activations quantized online to NVFP4 (computed s_g), the product against
    the oracle's NVFP4 activations times the oracle's MXFP4 weights."""
    import torch
    rng = np.random.default_rng(M + N + K)
    x = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qw, sw, _ = orc.quantize(w, orc.MXFP4)
    W_nv = fp4.mx_to_nv(upload(orc, qw, sw, 1.0))
    c = fp4.linear(to_dev_bf16(x), W_nv, fp4.FP4_NVFP4, out_dtype=0, weights_static=True)
    torch.cuda.synchronize()
    fp4.check_device_status()
    qa, sa, ga = orc.quantize(x, orc.NVFP4)
    ah = orc.dequantize(qa, sa, ga, orc.NVFP4)
    wh = orc.dequantize(qw, sw, 1.0, orc.MXFP4)
    ref, bound = orc.gemm_ref(ah, wh)
    err = np.abs(to_np(c).astype(np.float64) - ref)
    assert np.all(err <= 1e-5 * bound), np.max(err / np.maximum(bound, 1e-30))
