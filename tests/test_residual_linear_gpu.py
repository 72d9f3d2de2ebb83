"""GPU parity of fp4_linear_residual: the decode product with the sparse
residual lane of "Portable FP4 quantization (TransFP4)" §2.3 Eq.(3) in the
activations.  With both operands rotated by the same H,

    C = Q(H x - P H x) (W H)_q^T + (P H x)(W H)_q^T,

P keeping the largest rotated value of every 32-value unit (bf16).  The
reference is the oracle's: fp4_quantize_residual's encoding of x,
dequantized with the lane added back (still rotated), times the oracle's
dequantized W, in fp64; acceptance |C - C_ref| <= 1e-5 * sum_k |a_k||w_k|
(plus half a bf16 ulp of C_ref for BF16 output).  The lane's product runs on
the tensor cores as extra activation rows holding exact terms of each
residual (see the kernel), so it is held to the same bound as the rest.
"""
import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

from helpers import to_dev_bf16, to_np

pytestmark = pytest.mark.gpu

MX, NV, MX16 = 0, 1, 2


@pytest.fixture(scope="module")
def fp4():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_microscaling_quantization_b200 import build
    build.build()
    import fp4_microscaling_quantization_b200 as m
    return m


def upload(orc, q, s, g):
    import torch
    return (torch.from_numpy(np.ascontiguousarray(q)).cuda(), torch.from_numpy(orc.scales_to_atoms(s)).cuda(),
            torch.tensor([g], dtype=torch.float32, device="cuda"))


def reference(orc, x, qw, sw, gw, fmt, hk, gscale=None):
    qa, sa, ga, res = orc.quantize_residual(x, fmt, hadamard_k=hk, gscale=gscale)
    ah = orc.dequantize_residual(qa, sa, ga, res, fmt)  # the lane added back, still rotated
    wh = orc.dequantize(qw, sw, gw, fmt)
    return orc.gemm_ref(ah, wh)


def check(c, ref, bound, bf16):
    err = np.abs(to_np(c.float()).astype(np.float64) - ref)
    tol = 1e-5 * bound + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{bad.shape[0]} outputs out of tolerance, first {bad[:3].tolist()}: "
                           f"err {err[tuple(bad[0])]} tol {tol[tuple(bad[0])]}")


# whole tiles (100 tiles), clusters of 8 / 4 / 2, few tiles (3: clusters of 8
# where fp4_linear would cut tiles), more tiles than SMs (one CTA per tile in
# waves), K tails
SHAPES = [(1, 12800, 512, 0), (16, 12800, 1024, 32), (16, 2048, 2048, 128), (5, 4096, 1024, 16),
          (3, 8192, 800, 32), (16, 384, 4096, 64), (4, 160 * 128, 512, 0)]


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
@pytest.mark.parametrize("M,N,K,hk", SHAPES)
def test_residual_product_matches_oracle(fp4, orc, fmt, M, N, K, hk):
    import torch
    a, w = inputs.decode_linear(M, N, K, seed=M + N + K + hk)
    qw, sw, gw = orc.quantize(w, fmt, hadamard_k=hk)
    W = upload(orc, qw, sw, gw)
    c = fp4.linear_residual(to_dev_bf16(a), W, fmt, hadamard_k=hk, out_dtype=fp4.FP4_OUT_F32)
    torch.cuda.synchronize()
    fp4.check_device_status()
    ref, bound = reference(orc, a, qw, sw, gw, fmt, hk)
    check(c, ref, bound, False)


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
def test_outlier_channels(fp4, orc, fmt):
    """Activations with 1% outlier channels x50 (the rotate workload's
    recipe), where the lane carries the outliers; BF16 output."""
    import torch
    M, N, K = 16, 4096, 4096
    x = inputs.rotate_acts(rows=M, cols=K, seed=9)
    _, w = inputs.decode_linear(1, N, K, seed=10)
    qw, sw, gw = orc.quantize(w, fmt, hadamard_k=32)
    c = fp4.linear_residual(to_dev_bf16(x), upload(orc, qw, sw, gw), fmt, hadamard_k=32)
    torch.cuda.synchronize()
    ref, bound = reference(orc, x, qw, sw, gw, fmt, 32)
    check(c, ref, bound, True)


def test_static_activation_scale(fp4, orc):
    import torch
    M, N, K = 8, 4096, 2048
    a, w = inputs.decode_linear(M, N, K, seed=21)
    qw, sw, gw = orc.quantize(w, NV)
    gA = 0.0031
    c = fp4.linear_residual(to_dev_bf16(a), upload(orc, qw, sw, gw), NV, out_dtype=fp4.FP4_OUT_F32,
                            gscale=torch.tensor([gA], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    ref, bound = reference(orc, a, qw, sw, gw, NV, 0, gscale=gA)
    check(c, ref, bound, False)


def test_one_value_units_carry_the_whole_product(fp4, orc):
    """Activations with one nonzero value per 32-value unit: the FP4 stream is
    all zeros and C is the lane's product alone, x W_q^T with x's bf16 values
    (exact terms), checked against numpy's fp64 product."""
    import torch
    M, N, K = 4, 2048, 1024
    rng = np.random.default_rng(4)
    xf = np.zeros((M, K), np.float32)
    for m in range(M):
        for u in range(K // 32):
            xf[m, 32 * u + rng.integers(0, 32)] = rng.laplace(0, 1) * 2.0 ** rng.integers(-6, 7)
    x = inputs.f32_to_bf16_bits(xf)
    _, w = inputs.decode_linear(1, N, K, seed=6)
    for fmt in (MX, NV, MX16):
        qw, sw, gw = orc.quantize(w, fmt)
        c = fp4.linear_residual(to_dev_bf16(x), upload(orc, qw, sw, gw), fmt, out_dtype=fp4.FP4_OUT_F32)
        torch.cuda.synchronize()
        wh = orc.dequantize(qw, sw, gw, fmt).astype(np.float64)
        xb = inputs.bf16_bits_to_f32(x).astype(np.float64)
        ref = xb @ wh.T
        bound = np.abs(xb) @ np.abs(wh).T
        check(c, ref, bound, False)


def test_unsupported_and_empty(fp4):
    import torch
    from fp4_microscaling_quantization_b200 import _lib
    x = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    W = fp4.quantize(torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda"), MX)
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.linear_residual(x, W, MX)
    assert ei.value.code == 2  # M above 16: the decode product only
    c = fp4.linear_residual(x[:0], W, MX)
    assert c.shape == (0, 256)


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_full_size(fp4, orc, fmt, N, K):
    """The decode workloads with the lane on, static weights, BF16 out:
    every output of M = 16 against the oracle."""
    import torch
    M = 16
    a, _ = inputs.decode_linear(M, 8, K)
    _, w = inputs.decode_linear(1, N, K)
    qw, sw, gw = orc.quantize(w, fmt)
    c = fp4.linear_residual(to_dev_bf16(a), upload(orc, qw, sw, gw), fmt, weights_static=True)
    torch.cuda.synchronize()
    fp4.check_device_status()
    ref, bound = reference(orc, a, qw, sw, gw, fmt, 0)
    check(c, ref, bound, True)
