"""GPU parity of fp4_gemm against the oracle's fp64 product of the
dequantized operands.

Acceptance per element: |C - C_ref| <= 1e-5 * sum_k |a_k||w_k| for FP32
output; BF16 output adds half a bf16 ulp, 2^-8 |C_ref|.  With unit scales
every product is a multiple of 1/4 and every partial sum is exact in FP32, so
C must then be bit-exact.
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


def torch_sms() -> int:
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count


def upload(orc, q, s_logical, g):
    import torch
    qd = torch.from_numpy(np.ascontiguousarray(q)).cuda()
    sd = torch.from_numpy(orc.scales_to_atoms(s_logical)).cuda()
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    return qd, sd, gd


def run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, fmt, out_dtype, ldc=None):
    import torch
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qw.shape[0]
    a = upload(orc, qa, sa, ga)
    w = upload(orc, qw, sw, gw)
    dt = torch.float32 if out_dtype == 0 else torch.bfloat16
    if ldc is None:
        out = full = None
    else:
        full = torch.full((M, ldc), float("nan"), dtype=dt, device="cuda")
        out = full[:, :N]
    c = fp4.gemm(a, w, M, N, K, fmt, out_dtype=out_dtype, out=out)
    torch.cuda.synchronize()
    fp4.check_device_status()
    if full is not None:
        assert torch.isnan(full[:, N:].float()).all(), "GEMM wrote outside the N columns"
    return to_np(c.float())


def reference(orc, qa, sa, ga, qw, sw, gw, fmt):
    ah = orc.dequantize(qa, sa, ga, fmt)
    wh = orc.dequantize(qw, sw, gw, fmt)
    return orc.gemm_ref(ah, wh)


def assert_close(c, ref, bound, out_dtype):
    tol = 1e-5 * bound + (2.0 ** -8 * np.abs(ref) if out_dtype == 1 else 0.0)
    err = np.abs(c.astype(np.float64) - ref)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{bad.shape[0]} elements out of tolerance, first {bad[:3].tolist()}: "
                           f"got {c[tuple(bad[0])]} want {ref[tuple(bad[0])]} tol {tol[tuple(bad[0])]}")


def rand_q(rng, rows, K):
    return rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)


def unit_scales(fmt, rows, K):
    block = 32 if fmt == 0 else 16
    return np.full((rows, K // block), 127 if fmt == 0 else 0x38, np.uint8)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(128, 256, 256), (128, 256, 1024), (256, 512, 512), (130, 300, 512)])
def test_unit_scale_exact(fp4, orc, fmt, shape):
    M, N, K = shape
    rng = np.random.default_rng(M + N + K + fmt)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = unit_scales(fmt, M, K), unit_scales(fmt, N, K)
    c = run_gemm(fp4, orc, qa, sa, 1.0, qw, sw, 1.0, fmt, 0)
    ref, _ = reference(orc, qa, sa, 1.0, qw, sw, 1.0, fmt)
    assert np.array_equal(c.astype(np.float64), ref)


@pytest.mark.parametrize("fmt", [0, 1])
def test_impulses_pin_operand_and_scale_layout(fp4, orc, fmt):
    """One nonzero element in A and W and one distinct scale per block: C
    lights exactly one entry, with the product of the two scales."""
    M, N, K = 256, 512, 512
    block = 32 if fmt == 0 else 16
    rng = np.random.default_rng(fmt)
    for trial in range(6):
        m, n, k = int(rng.integers(M)), int(rng.integers(N)), int(rng.integers(K))
        qa = np.zeros((M, K // 2), np.uint8)
        qw = np.zeros((N, K // 2), np.uint8)
        qa[m, k // 2] = (3 if k % 2 == 0 else 3 << 4)          # 1.5
        qw[n, k // 2] = (0xD if k % 2 == 0 else 0xD << 4)      # -3
        if fmt == 0:
            sa = rng.integers(120, 135, (M, K // block)).astype(np.uint8)
            sw = rng.integers(120, 135, (N, K // block)).astype(np.uint8)
        else:
            sa = rng.integers(0x20, 0x60, (M, K // block)).astype(np.uint8)
            sw = rng.integers(0x20, 0x60, (N, K // block)).astype(np.uint8)
        c = run_gemm(fp4, orc, qa, sa, 1.0, qw, sw, 1.0, fmt, 0)
        ref, _ = reference(orc, qa, sa, 1.0, qw, sw, 1.0, fmt)
        nz = np.argwhere(c != 0)
        assert nz.tolist() == [[m, n]], (trial, nz[:4].tolist(), (m, n, k))
        assert c[m, n] == ref[m, n]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("out_dtype", [0, 1])
@pytest.mark.parametrize("shape", [(128, 256, 512), (200, 520, 1024), (1, 8, 256), (16, 4096, 512), (300, 256, 2048)])
def test_random_scales_within_tolerance(fp4, orc, fmt, out_dtype, shape):
    M, N, K = shape
    rng = np.random.default_rng(M * 3 + N + K)
    va = rng.laplace(0, 1, (M, K)).astype(np.float32)
    va[rng.random((M, K)) < 0.01] *= 20
    vw = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    qa, sa, ga = orc.quantize(inputs.f32_to_bf16_bits(va), fmt)
    qw, sw, gw = orc.quantize(inputs.f32_to_bf16_bits(vw), fmt)
    c = run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, fmt, out_dtype)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(c, ref, bound, out_dtype)


def test_tiny_linear_workload(fp4, orc):
    """MXFP4 W4A4 linear, tiny: A 128x512, W 256x512, full brute force."""
    a, w = inputs.tiny_linear()
    qa, sa, ga = orc.quantize(a, 0)
    qw, sw, gw = orc.quantize(w, 0)
    for out_dtype in (0, 1):
        c = run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, 0, out_dtype)
        ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, 0)
        assert_close(c, ref, bound, out_dtype)


@pytest.mark.parametrize("fmt", [0, 1])
def test_strided_output(fp4, orc, fmt):
    M, N, K = 130, 264, 512
    rng = np.random.default_rng(5)
    qa, sa, ga = orc.quantize(inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32)), fmt)
    qw, sw, gw = orc.quantize(inputs.f32_to_bf16_bits(rng.laplace(0, 1, (N, K)).astype(np.float32)), fmt)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    for out_dtype, ldc in ((0, 300), (1, 304), (1, 270)):
        c = run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, fmt, out_dtype, ldc=ldc)
        assert_close(c, ref, bound, out_dtype)


@pytest.mark.parametrize("fmt", [0, 1])
def test_rotated_operands_preserve_product(fp4, orc, fmt):
    """(X H)(W H)^T = X W^T: quantizing both operands with the same H_k gives
    the product of the unrotated tensors up to quantization error."""
    import torch
    M, N, K = 128, 256, 1024
    a = inputs.rotate_acts(rows=M, cols=K, seed=8)
    rng = np.random.default_rng(9)
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    exact = inputs.bf16_bits_to_f32(a).astype(np.float64) @ inputs.bf16_bits_to_f32(w).astype(np.float64).T
    errs = {}
    for hk in (0, 128):
        A = fp4.quantize(to_dev_bf16(a), fmt, hadamard_k=hk)
        W = fp4.quantize(to_dev_bf16(w), fmt, hadamard_k=hk)
        c = to_np(fp4.gemm(A, W, M, N, K, fmt, out_dtype=0)).astype(np.float64)
        torch.cuda.synchronize()
        # the GEMM over the rotated operands equals the oracle product of their dequantized values
        qa, sa, ga = orc.quantize(a, fmt, hadamard_k=hk)
        qw, sw, gw = orc.quantize(w, fmt, hadamard_k=hk)
        ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
        assert_close(c, ref, bound, 0)
        errs[hk] = np.linalg.norm(c - exact) / np.linalg.norm(exact)
    assert errs[128] < 0.25 and errs[0] < 0.5
    if fmt == 0:
        # MXFP4: the rotation spreads the outlier channels and lowers the error.
        # (For NVFP4 the pages report rotation can raise the error a little,
        # which is what this workload shows too, so no ordering is asserted.)
        assert errs[128] < errs[0]


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_full_size_prefill_sampled(fp4, orc, fmt):
    """8192 x 8192 activations times a 28672 x 8192 weight (70B MLP shape), in
    the benchmark's launch configuration; 64 x 64 sampled outputs against the
    oracle's fp64 product of the same quantized bytes.  Formats: MXFP4, NVFP4
    and MXFP4 on 16-element blocks (the benchmark's three prefill rows)."""
    import torch
    M, N, K = 8192, 28672, 8192
    a, w = inputs.prefill_linear()
    A = fp4.quantize(to_dev_bf16(a), fmt)
    W = fp4.quantize(to_dev_bf16(w), fmt)
    del a
    c = fp4.gemm(A, W, M, N, K, fmt, out_dtype=1)
    torch.cuda.synchronize()
    fp4.check_device_status()
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(M, 64, replace=False))
    cols = np.sort(rng.choice(N, 64, replace=False))
    block = 32 if fmt == 0 else 16
    nkb = K // block

    def deq(T, idx, nrows):
        q = to_np(T[0])[idx]
        s_log = orc.scales_from_atoms(to_np(T[1]), nrows, nkb)[idx]
        return orc.dequantize(q, s_log, float(to_np(T[2])[0]), fmt)

    ah, wh = deq(A, rows, M), deq(W, cols, N)
    ref, bound = orc.gemm_ref(ah, wh)
    got = to_np(c.float())[np.ix_(rows, cols)]
    assert_close(got, ref, bound, 1)
    del c, A, W
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ decode ----
DECODE_SHAPES = [(1, 4096, 512), (4, 1000, 768), (16, 4096, 1024), (3, 40000, 256), (2, 20000, 512),
                 (16, 300, 4096), (7, 8, 256)]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("out_dtype", [0, 1])
@pytest.mark.parametrize("shape", DECODE_SHAPES)
def test_decode_within_tolerance(fp4, orc, fmt, out_dtype, shape):
    """M <= 16 takes the weight-streaming split-K kernel.  On 148 SMs the
    shapes cover every work split: cluster splits of 2 and 4 CTAs per tile
    ((1, 4096, 512), (16, 4096, 1024)), global splits summed by the reduction
    kernel ((4, 1000, 768), (16, 300, 4096) with a ragged last tile), stream-K
    with whole tiles only, three segments per CTA ((3, 40000, 256)), stream-K
    with tiles cut between CTAs ((2, 20000, 512)) and a single CTA
    ((7, 8, 256)).  The workspace is needed exactly when partials go through
    global memory."""
    M, N, K = shape
    rng = np.random.default_rng(M + N + K)
    qa, sa, ga = orc.quantize(inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32)), fmt)
    qw, sw, gw = orc.quantize(inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32)), fmt)
    if torch_sms() == 148:
        needs_ws = shape in ((4, 1000, 768), (16, 300, 4096), (2, 20000, 512))
        assert (fp4.gemm_workspace_size(M, N, K, fmt) > 0) == needs_ws
    c = run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, fmt, out_dtype)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(c, ref, bound, out_dtype)


@pytest.mark.parametrize("fmt", [0, 1])
def test_decode_unit_scale_exact_and_deterministic(fp4, orc, fmt):
    import torch
    M, N, K = 16, 2048, 2048
    rng = np.random.default_rng(3)
    qa, qw = rand_q(rng, M, K), rand_q(rng, N, K)
    sa, sw = unit_scales(fmt, M, K), unit_scales(fmt, N, K)
    c1 = run_gemm(fp4, orc, qa, sa, 1.0, qw, sw, 1.0, fmt, 0)
    c2 = run_gemm(fp4, orc, qa, sa, 1.0, qw, sw, 1.0, fmt, 0)
    ref, _ = reference(orc, qa, sa, 1.0, qw, sw, 1.0, fmt)
    assert np.array_equal(c1.astype(np.float64), ref)
    assert np.array_equal(c1.view(np.uint32), c2.view(np.uint32))


def test_decode_workspace_checked(fp4, orc):
    import torch
    M, N, K = 4, 1024, 512
    need = fp4.gemm_workspace_size(M, N, K, 0)
    qa = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.zeros((128 * K // 32,), dtype=torch.uint8, device="cuda")
    qw = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.zeros((N * K // 32,), dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    small = torch.empty((need - 16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(fp4.Fp4Error):
        fp4.gemm((qa, sa, g), (qw, sw, g), M, N, K, 0, workspace=small)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("NK", [(14336, 4096), (4096, 14336)])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_full_size_decode(fp4, orc, fmt, NK, M):
    """Decode shapes of the 8B MLP: every output against the oracle."""
    N, K = NK
    a, w = inputs.decode_linear(M, N, K)
    qa, sa, ga = orc.quantize(a, fmt)
    qw, sw, gw = orc.quantize(w, fmt)
    c = run_gemm(fp4, orc, qa, sa, ga, qw, sw, gw, fmt, 1)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(c, ref, bound, 1)


# ------------------------------------------------------------------ linear ----
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,hk", [(1, 0), (16, 64), (5, 128), (200, 32)])
def test_linear_online_activation_quantization(fp4, orc, fmt, M, hk):
    """fp4_linear = online quantization of bf16 activations + the GEMM; the
    reference quantizes the same activations with the oracle."""
    import torch
    N, K = 1024, 1024
    rng = np.random.default_rng(M + hk)
    x = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qw, sw, gw = orc.quantize(w, fmt, hadamard_k=hk)
    W = upload(orc, qw, sw, gw)
    c = fp4.linear(to_dev_bf16(x), W, fmt, hadamard_k=hk, out_dtype=0)
    torch.cuda.synchronize()
    qa, sa, ga = orc.quantize(x, fmt, hadamard_k=hk)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, fmt)
    assert_close(to_np(c), ref, bound, 0)


@pytest.mark.parametrize("N,K", [(512, 512), (4096, 2048)])
def test_linear_static_activation_scale(fp4, orc, N, K):
    """A given activation tensor scale, with a global split (4 tiles) and a
    cluster split (32 tiles) of the decode product."""
    import torch
    M = 8
    rng = np.random.default_rng(0)
    x = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    qw, sw, gw = orc.quantize(w, 1)
    W = upload(orc, qw, sw, gw)
    gA = 0.004
    c = fp4.linear(to_dev_bf16(x), W, 1, out_dtype=0, gscale=torch.tensor([gA], device="cuda"))
    torch.cuda.synchronize()
    qa, sa, ga = orc.quantize(x, 1, gscale=gA)
    ref, bound = reference(orc, qa, sa, ga, qw, sw, gw, 1)
    assert_close(to_np(c), ref, bound, 0)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,N,K,hk", [(16, 14336, 4096, 0), (4, 4096, 14336, 0), (3, 40000, 256, 0),
                                      (2, 20000, 512, 0), (1, 300, 4096, 32), (16, 2048, 2048, 128),
                                      (5, 14336, 1024, 64), (8, 4096, 2048, 32), (16, 14336, 512, 16)])
def test_linear_decode_fused_reduction_matches_gemm(fp4, orc, fmt, M, N, K, hk):
    """fp4_linear's decode path (one-cluster activation quantizer + split-K,
    with partials of a globally split tile summed by the last CTA of the tile)
    gives bit-identical results to fp4_quantize + fp4_gemm (separate reduction
    kernel): the partial sums are added in the same CTA order.  Whole tiles,
    cluster splits and global splits, every rotation size and M from 1 to 16
    are exercised; repeated calls are identical."""
    import torch
    a, w = inputs.decode_linear(M, N, K, seed=N + K)
    xd = to_dev_bf16(a)
    W = fp4.quantize(to_dev_bf16(w), fmt, hadamard_k=hk)
    A = fp4.quantize(xd, fmt, hadamard_k=hk)
    ref = fp4.gemm(A, W, M, N, K, fmt, out_dtype=0)
    c1 = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=0)
    c2 = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert torch.equal(c1.view(torch.int32), ref.view(torch.int32))
    assert torch.equal(c1.view(torch.int32), c2.view(torch.int32))
    # bf16 output of the fused path equals the rounding of the fp32 one
    cb = fp4.linear(xd, W, fmt, hadamard_k=hk, out_dtype=1)
    torch.cuda.synchronize()
    assert torch.equal(cb, c1.to(torch.bfloat16))


@pytest.mark.parametrize("fmt", [0, 1])
def test_linear_static_weights_chain(fp4, orc, fmt):
    """weights_static lets the decode kernel stream W while the previous
    kernel in the stream finishes; activations and outputs stay ordered.  A
    chain of dependent decode layers (each output is the next layer's input,
    N = K) with a different weight per layer, issued back to back without a
    synchronisation, equals the same chain without the option bit for bit."""
    import torch
    M, D, L = 4, 4096, 6
    rng = np.random.default_rng(17 + fmt)
    Ws = []
    for i in range(L):
        w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (D, D)).astype(np.float32))
        Ws.append(fp4.quantize(to_dev_bf16(w), fmt))
    x0 = to_dev_bf16(inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, D)).astype(np.float32)))
    ws = torch.empty((fp4.linear_workspace_size(M, D, D, fmt),), dtype=torch.uint8, device="cuda")

    def chain(static):
        outs, x = [], x0
        for i in range(L):
            x = fp4.linear(x, Ws[i], fmt, out_dtype=1, workspace=ws, weights_static=static)
            outs.append(x)
        torch.cuda.synchronize()
        fp4.check_device_status()
        return outs

    ref = chain(False)
    for _ in range(3):
        got = chain(True)
        for i in range(L):
            assert torch.equal(got[i], ref[i]), f"layer {i} differs"
