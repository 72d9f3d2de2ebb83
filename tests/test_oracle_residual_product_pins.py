"""Pins of the oracle's reference for the decode product with the sparse
residual lane ("Portable FP4 quantization (TransFP4)" §2.3 Eq.(3)):
C_ref = (Q(Hx - PHx) + PHx) (WH)_q^T in fp64, composed from
quantize_residual, dequantize_residual (kept in the rotated domain) and
gemm_ref.  It is pinned against numbers built without the oracle's lane code:

- lane off: with every residual word zeroed, the product is that of the FP4
  stream alone;
- the decomposition: the product minus the stream's product is R W_q^T,
  with R built here by numpy from x itself (in every 32-value unit, the
  first value of largest magnitude, rounded to bf16 by torch);
- one nonzero value per unit: the stream is empty and the product is
  numpy's fp64 x W_q^T of the bf16 activations.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs


def stream_and_lane(orc, x, fmt):
    q, s, g, res = orc.quantize_residual(x, fmt)
    with_lane = orc.dequantize_residual(q, s, g, res, fmt)
    stream = orc.dequantize(q, s, g, fmt)
    return q, s, g, res, with_lane, stream


def numpy_lane(x_bits):
    """R: in every 32-value unit the first value of largest magnitude, bf16
    (x is bf16 already, so the value is exact), zeros elsewhere."""
    import torch
    xf = inputs.bf16_bits_to_f32(x_bits)
    rows, cols = xf.shape
    u = xf.reshape(rows, cols // 32, 32)
    idx = np.argmax(np.abs(u), axis=2)  # first of equal ones
    R = np.zeros_like(u)
    r_, c_ = np.meshgrid(np.arange(rows), np.arange(cols // 32), indexing="ij")
    vals = torch.from_numpy(u[r_, c_, idx].copy()).to(torch.bfloat16).float().numpy()
    R[r_, c_, idx] = vals
    return R.reshape(rows, cols)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_lane_off_is_the_stream_product(orc, fmt):
    a, w = inputs.decode_linear(5, 96, 512, seed=30 + fmt)
    qw, sw, gw = orc.quantize(w, fmt)
    wh = orc.dequantize(qw, sw, gw, fmt)
    q, s, g, res, _, stream = stream_and_lane(orc, a, fmt)
    off = orc.dequantize_residual(q, s, g, np.zeros_like(res), fmt)
    c_off, _ = orc.gemm_ref(off, wh)
    c_stream, _ = orc.gemm_ref(stream, wh)
    assert np.array_equal(c_off, c_stream)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_decomposition_against_numpy_lane(orc, fmt):
    a, w = inputs.decode_linear(7, 64, 1024, seed=40 + fmt)
    qw, sw, gw = orc.quantize(w, fmt)
    wh = orc.dequantize(qw, sw, gw, fmt).astype(np.float64)
    _, _, _, _, with_lane, stream = stream_and_lane(orc, a, fmt)
    R = numpy_lane(a)
    assert np.array_equal(with_lane.astype(np.float64) - stream.astype(np.float64), R.astype(np.float64))
    c, bound = orc.gemm_ref(with_lane, wh)
    c_stream, _ = orc.gemm_ref(stream, wh)
    lane_prod = R.astype(np.float64) @ wh.T
    assert np.all(np.abs((c - c_stream) - lane_prod) <= 1e-12 * bound)


def test_one_value_units(orc):
    rng = np.random.default_rng(12)
    M, N, K = 3, 48, 256
    xf = np.zeros((M, K), np.float32)
    for m in range(M):
        for u in range(K // 32):
            xf[m, 32 * u + rng.integers(0, 32)] = rng.laplace(0, 1) * 2.0 ** rng.integers(-8, 9)
    x = inputs.f32_to_bf16_bits(xf)
    _, w = inputs.decode_linear(1, N, K, seed=13)
    for fmt in (0, 1, 2):
        qw, sw, gw = orc.quantize(w, fmt)
        wh = orc.dequantize(qw, sw, gw, fmt).astype(np.float64)
        _, _, _, _, with_lane, stream = stream_and_lane(orc, x, fmt)
        assert not np.any(stream)
        c, bound = orc.gemm_ref(with_lane, wh)
        ref = inputs.bf16_bits_to_f32(x).astype(np.float64) @ wh.T
        assert np.all(np.abs(c - ref) <= 1e-12 * bound)
