"""Failure detection without faulting the GPU: a test hook makes the next
GEMM launch's producer issue no loads, so the MMA warp's bounded mbarrier
wait runs out (short budget).  The kernel must return (no hang), store
nothing, free its tensor memory, and report FP4_ERR_TIMEOUT through
fp4_check_device_status; the next call must work normally."""
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


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (256, 512, 512), (4, 1024, 512)])
def test_bounded_wait_reports_timeout_and_recovers(fp4, M, N, K):
    import torch
    from fp4_microscaling_quantization_b200 import _lib
    rng = np.random.default_rng(M + N)
    a = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    A = fp4.quantize(to_dev_bf16(a), 0)
    W = fp4.quantize(to_dev_bf16(w), 0)
    ref = fp4.gemm(A, W, M, N, K, 0, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()

    sentinel = torch.full((M, N), 12345.0, dtype=torch.float32, device="cuda")
    assert _lib.lib().fp4_test_inject_stall(1, 50_000_000) == 0   # 50 ms budget
    fp4.gemm(A, W, M, N, K, 0, out_dtype=0, out=sentinel)
    torch.cuda.synchronize()
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.check_device_status()
    assert ei.value.code == 5  # FP4_ERR_TIMEOUT
    if 16 < M <= 128:
        # the single-CTA tiled kernel stores nothing after giving up
        assert torch.all(sentinel == 12345.0)

    again = fp4.gemm(A, W, M, N, K, 0, out_dtype=0)
    torch.cuda.synchronize()
    fp4.check_device_status()  # cleared, and the new call is clean
    assert torch.equal(again, ref)


@pytest.mark.parametrize("M,out_fmt", [(128, 0), (256, 1)])
def test_quantizing_epilogue_times_out_and_recovers(fp4, M, out_fmt):
    """The same for the GEMM whose epilogue quantizes C (fp4_gemm_quantized)."""
    import torch
    from fp4_microscaling_quantization_b200 import _lib
    N, K = 256, 512
    rng = np.random.default_rng(M + 7)
    a = inputs.f32_to_bf16_bits(rng.laplace(0, 1, (M, K)).astype(np.float32))
    w = inputs.f32_to_bf16_bits(rng.laplace(0, 0.02, (N, K)).astype(np.float32))
    A = fp4.quantize(to_dev_bf16(a), 0)
    W = fp4.quantize(to_dev_bf16(w), 0)
    gC = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    ref = fp4.gemm_quantized(A, W, M, N, K, 0, out_fmt, gscale=gC if out_fmt else None)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert _lib.lib().fp4_test_inject_stall(1, 50_000_000) == 0
    fp4.gemm_quantized(A, W, M, N, K, 0, out_fmt, gscale=gC if out_fmt else None)
    torch.cuda.synchronize()
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.check_device_status()
    assert ei.value.code == 5
    again = fp4.gemm_quantized(A, W, M, N, K, 0, out_fmt, gscale=gC if out_fmt else None)
    torch.cuda.synchronize()
    fp4.check_device_status()
    assert torch.equal(again[0], ref[0]) and torch.equal(again[1], ref[1])
