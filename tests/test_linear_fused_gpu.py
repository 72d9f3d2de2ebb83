"""GPU parity of fp4_linear's single-launch decode path (M <= 16): the decode
kernel quantizes the bf16 activations itself ("4.5 FP8 and NVFP4/MXFP4"
§4.2, online quantization; "FP4 quantization analysis: MXFP4 vs NVFP4"
§3.2.3, online rotation) into its pipeline stages, then runs the block-scaled
product ("4.5 FP8 and NVFP4/MXFP4" §5).

- Bit-identity with fp4_quantize + fp4_gemm: the activations are encoded by
  the quantize kernels' own per-unit encoder and the product adds the same
  partials in the same order, so every format, rotation size, rounding
  option, tail and work split (whole tiles; clusters of 2 to 8 CTAs, whose
  CTAs also combine the NVFP4 tensor maximum) must agree bit for bit.
- The full decode workloads (W 14336 x 4096 and 4096 x 14336, M = 1, 4, 16,
  static weights as the benchmark calls them), every output against the
  oracle's fp64 product within 1e-5 * sum_k |a_k||w_k|.
- The bounded waits: a stalled launch reports FP4_ERR_TIMEOUT and the next
  call is clean.
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


def sms():
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count


def split_of(N, K):
    """The decode work split the library picks (whole tiles, a cluster of
    CTAs per tile, or a global split), restated from its plan: 128-row W
    tiles, 256-wide K steps, clusters of at most 8."""
    n = sms()
    ntiles, nk = -(-N // 128), -(-K // 256)
    if ntiles > n or ntiles * 16 <= n:
        return "global"
    split = 1
    while split * 2 <= 8 and ntiles * split * 2 <= n and split * 2 <= nk:
        split *= 2
    return "whole" if split == 1 else f"cluster{split}"


def gemm_path(fp4, xd, W, fmt, hk, out_dtype, round_, rule, gA=None):
    """fp4_quantize + fp4_gemm with the same options."""
    M, K = xd.shape
    N = W[0].shape[0]
    A = fp4.quantize(xd, fmt, hadamard_k=hk, round=round_, mx_scale_rule=rule, gscale=gA)
    return fp4.gemm(A, W, M, N, K, fmt, out_dtype=out_dtype)


# (M, N, K, hk): whole tiles (N = 12800: 100 tiles), clusters of 8 (16 tiles,
# K = 2048), of 4 (32 tiles, K = 1024) and of 2 (64 tiles), a K tail (800 =
# 3 steps + 32), every rotation size, and whole tiles whose 32 / 25 K steps
# run through the 8-stage pipeline four times.
SHAPES = [(1, 12800, 512, 0), (16, 12800, 512, 128), (7, 12800, 800, 32), (16, 2048, 2048, 0), (3, 2048, 2048, 64),
          (16, 4096, 1024, 16), (4, 4096, 800, 32), (16, 8192, 512, 128), (9, 8192, 4096, 64),
          (4, 12800, 8192, 0), (16, 12800, 6400, 32)]


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
@pytest.mark.parametrize("M,N,K,hk", SHAPES)
def test_single_launch_matches_quantize_then_gemm(fp4, fmt, M, N, K, hk):
    import torch
    assert split_of(N, K) != "global"
    a, w = inputs.decode_linear(M, N, K, seed=M * 7 + N + K + hk)
    xd = to_dev_bf16(a)
    W = fp4.quantize(to_dev_bf16(w), fmt, hadamard_k=hk)
    launches0 = fp4.kernel_launches()
    c = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=0)
    launches = fp4.kernel_launches() - launches0
    ref = gemm_path(fp4, xd, W, fmt, hk, 0, 0, 0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert launches == 1, f"{launches} launches for one decode linear"
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    cb = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=1)
    torch.cuda.synchronize()
    assert torch.equal(cb, ref.to(torch.bfloat16))


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
@pytest.mark.parametrize("round_,rule", [(1, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("M,N,K,hk", [(5, 12800, 512, 32), (16, 4096, 1024, 0)])
def test_rounding_options(fp4, fmt, round_, rule, M, N, K, hk):
    """Ties away from zero and the FLOOR exponent rule reach the fused encoder."""
    import torch
    a, w = inputs.decode_linear(M, N, K, seed=11 + M)
    xd = to_dev_bf16(a)
    W = fp4.quantize(to_dev_bf16(w), fmt, hadamard_k=hk)
    c = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=0, round=round_, mx_scale_rule=rule)
    ref = gemm_path(fp4, xd, W, fmt, hk, 0, round_, rule)
    torch.cuda.synchronize()
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("M,N,K", [(4, 12800, 512), (16, 2048, 2048)])
def test_static_activation_scale(fp4, M, N, K):
    """NVFP4 with the caller's activation tensor scale (no tensor maximum)."""
    import torch
    a, w = inputs.decode_linear(M, N, K, seed=3)
    xd = to_dev_bf16(a)
    W = fp4.quantize(to_dev_bf16(w), NV)
    gA = torch.tensor([0.0037], dtype=torch.float32, device="cuda")
    c = fp4.linear(xd, W, NV, out_dtype=0, gscale=gA)
    ref = gemm_path(fp4, xd, W, NV, 0, 0, 0, 0, gA=gA)
    torch.cuda.synchronize()
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("M,N,K", [(4, 2048, 2048), (16, 2048, 10240)])
def test_zero_and_single_outlier_activations(fp4, M, N, K):
    """All-zero activations give C = 0 (NVFP4 s_g = 1, zero scales); one
    nonzero activation sets the tensor maximum of every CTA of a cluster
    split: each CTA reads all of x (16 KB of x), or the CTAs exchange their
    K slices' maxima (320 KB), including those whose slice holds only
    zeros."""
    import torch
    _, w = inputs.decode_linear(1, N, K, seed=5)
    for fmt in (MX, NV, MX16):
        W = fp4.quantize(to_dev_bf16(w), fmt)
        x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        c = fp4.linear(x, W, fmt, out_dtype=0)
        torch.cuda.synchronize()
        assert torch.count_nonzero(c) == 0
        x[2, K - 7] = 3.5
        c = fp4.linear(x, W, fmt, out_dtype=0)
        ref = gemm_path(fp4, x, W, fmt, 0, 0, 0, 0)
        torch.cuda.synchronize()
        assert torch.equal(c.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("M,N,K", [(4, 12800, 512), (4, 4096, 1024)])
def test_stalled_launch_times_out_and_recovers(fp4, M, N, K):
    """Failure detection of the single-launch path: with the test hook the
    weight loads are never issued, every bounded wait gives up (the
    activation quantizers included), the call reports FP4_ERR_TIMEOUT through
    fp4_check_device_status, and the next call matches the reference."""
    import torch
    from fp4_microscaling_quantization_b200 import _lib
    a, w = inputs.decode_linear(M, N, K, seed=8)
    xd = to_dev_bf16(a)
    W = fp4.quantize(to_dev_bf16(w), NV)
    ref = gemm_path(fp4, xd, W, NV, 0, 0, 0, 0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert _lib.lib().fp4_test_inject_stall(1, 50_000_000) == 0
    fp4.linear(xd, W, NV, out_dtype=0)
    torch.cuda.synchronize()
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.check_device_status()
    assert ei.value.code == 5
    again = fp4.linear(xd, W, NV, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert torch.equal(again.view(torch.int32), ref.view(torch.int32))


# ------------------------------------------------------------ full size -----
def oracle_ref(orc, x, qw, sw, gw, fmt, w_fmt=None):
    w_fmt = fmt if w_fmt is None else w_fmt
    qa, sa, ga = orc.quantize(x, fmt)
    return orc.gemm_ref(orc.dequantize(qa, sa, ga, fmt), orc.dequantize(qw, sw, gw, w_fmt))


def check(c, ref, bound):
    err = np.abs(to_np(c.float()).astype(np.float64) - ref)
    tol = 1e-5 * bound + 2.0 ** -8 * np.abs(ref)  # BF16 output
    bad = np.argwhere(err > tol)
    assert bad.size == 0, f"{bad.shape[0]} outputs out of tolerance, first {bad[:3].tolist()}"


@pytest.mark.parametrize("fmt", [MX, NV, MX16])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_full_size_static_weights(fp4, orc, fmt, N, K):
    """The benchmarked decode call (fp4_linear, weights_static, BF16 out) on
    the full decode workloads, M = 1, 4, 16: every output against the oracle."""
    import torch
    _, w = inputs.decode_linear(1, N, K)
    qw, sw, gw = orc.quantize(w, fmt)
    W = (torch.from_numpy(np.ascontiguousarray(qw)).cuda(), torch.from_numpy(orc.scales_to_atoms(sw)).cuda(),
         torch.tensor([gw], dtype=torch.float32, device="cuda"))
    for M in (1, 4, 16):
        a, _ = inputs.decode_linear(M, 8, K)
        c = fp4.linear(to_dev_bf16(a), W, fmt, weights_static=True)
        torch.cuda.synchronize()
        fp4.check_device_status()
        ref, bound = oracle_ref(orc, a, qw, sw, gw, fmt)
        check(c, ref, bound)


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_full_size_nvfp4_activations_mxfp4_weights(fp4, orc, N, K):
    """The workload's literal reading at full size: NVFP4 activations
    quantized online against MXFP4 weights bound once to the NVFP4 form."""
    import torch
    _, w = inputs.decode_linear(1, N, K)
    qw, sw, _ = orc.quantize(w, orc.MXFP4)
    W_mx = (torch.from_numpy(np.ascontiguousarray(qw)).cuda(), torch.from_numpy(orc.scales_to_atoms(sw)).cuda(),
            torch.ones((1,), dtype=torch.float32, device="cuda"))
    W_nv = fp4.mx_to_nv(W_mx)
    for M in (1, 4, 16):
        a, _ = inputs.decode_linear(M, 8, K)
        c = fp4.linear(to_dev_bf16(a), W_nv, NV, weights_static=True)
        torch.cuda.synchronize()
        fp4.check_device_status()
        ref, bound = oracle_ref(orc, a, qw, sw, 1.0, NV, w_fmt=orc.MXFP4)
        check(c, ref, bound)
