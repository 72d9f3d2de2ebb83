"""GPU parity of the sparse residual lane ("Portable FP4 quantization
(TransFP4)" §2.3 Eq.(3), one value per 32): packed nibbles, scale bytes, the
NVFP4 tensor scale and the residual words (bf16 bits | index << 16) are
bit-exact against the oracle, and so is the dequantized fp32 tensor (bf16
output: its RNE rounding).
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import bf16_tensor_bits, to_dev_bf16, to_np

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


def check(fp4, orc, x, fmt, hk=0, tie=0, gscale=None):
    import torch
    gs = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    q, s, g, res = fp4.quantize_residual(to_dev_bf16(x), fmt, hadamard_k=hk, round=tie, gscale=gs)
    torch.cuda.synchronize()
    oq, os_, og, ores = orc.quantize_residual(x, fmt, hadamard_k=hk, tie=tie, gscale=gscale)
    assert np.array_equal(to_np(q), oq), "nibbles differ"
    assert np.array_equal(to_np(s), orc.scales_to_atoms(os_)), "scales differ"
    assert np.array_equal(to_np(res).view(np.uint32), ores), "residual words differ"
    if fmt == 1:
        assert np.float32(to_np(g)[0]) == np.float32(og)
    return (q, s, g, res), (oq, os_, og, ores)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hk", [0, 16, 32, 64, 128])
@pytest.mark.parametrize("shape", [(1, 128), (37, 3104), (130, 1024)])
def test_residual_quantize_parity(fp4, orc, fmt, hk, shape):
    rows, cols = shape
    if hk and cols % hk:
        pytest.skip("cols not a multiple of k")
    x = inputs.f32_to_bf16_bits(inputs.table5_activation(rows * cols, seed=rows + hk).reshape(rows, cols))
    check(fp4, orc, x, fmt, hk=hk)


@pytest.mark.parametrize("fmt,tie,gscale", [(0, 1, None), (1, 1, None), (1, 0, 0.01), (1, 0, 1e-30)])
def test_residual_modes(fp4, orc, fmt, tie, gscale):
    x = inputs.quant_sweep(rows=40, cols=2048, seed=19)
    check(fp4, orc, x, fmt, hk=32, tie=tie, gscale=gscale)


def test_residual_ties_and_special_units(fp4, orc):
    """Units of equal magnitudes (the first index wins), zeros, a lone value,
    negative maxima and values near the bf16 maximum."""
    rows = []
    rows.append(np.full(64, -2.0, np.float32))
    rows.append(np.zeros(64, np.float32))
    r = np.zeros(64, np.float32)
    r[7] = 3.0
    r[40] = -1e-3
    rows.append(r)
    rows.append(np.tile(np.array([1, -1], np.float32), 32))
    rows.append(np.linspace(-3e38, 3e38, 64).astype(np.float32))
    x = inputs.f32_to_bf16_bits(np.stack(rows))
    for fmt in (0, 1):
        for tie in (0, 1):
            check(fp4, orc, x, fmt, tie=tie)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hk", [0, 32])
@pytest.mark.parametrize("bf16", [0, 1])
def test_residual_dequantize_parity(fp4, orc, fmt, hk, bf16):
    import torch
    x = inputs.f32_to_bf16_bits(inputs.table5_activation(130 * 512, seed=4).reshape(130, 512))
    (q, s, g, res), (oq, os_, og, ores) = check(fp4, orc, x, fmt, hk=hk)
    out = fp4.dequantize_residual(q, s, g, res, fmt, hadamard_k=hk, out_dtype=bf16)
    torch.cuda.synchronize()
    ref = orc.dequantize_residual(oq, os_, og, ores, fmt, hadamard_k=hk)
    if bf16:
        assert np.array_equal(bf16_tensor_bits(out), inputs.f32_to_bf16_bits(ref))
    else:
        assert np.array_equal(to_np(out).view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_residual_full_size(fp4, orc, fmt):
    """1024 x 131072 heavy-tailed tensor with a 32-point rotation: whole-tensor
    parity, and the lane's reconstruction error below the rotation alone."""
    import torch
    x = inputs.quant_sweep()
    (q, s, g, res), (oq, os_, og, ores) = check(fp4, orc, x, fmt, hk=32)
    xs = inputs.bf16_bits_to_f32(x[:16])
    lane = orc.nmse(xs, orc.dequantize_residual(oq[:16], os_[:16], og, ores[:16], fmt, hadamard_k=32))
    pq, ps, pg = orc.quantize(x[:16], fmt, hadamard_k=32, gscale=og if fmt else None)
    plain = orc.nmse(xs, orc.dequantize(pq, ps, pg, fmt, hadamard_k=32))
    assert lane < plain
    del q, s, g, res
    torch.cuda.empty_cache()
