"""GPU check of fp4_gemm_decode_noalloc, the decode GEMM for callers that
cannot allocate device memory when they call it (for example code running
inside a stream capture, or a plugin handed fixed buffers): its split-K
partials live in a fixed array inside the library instead of a workspace.

It is called through the C ABI and compared with fp4_gemm (the entry point
that takes a caller workspace) on two calls in a row, within the GEMM
tolerance the other tests use.  Collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from fp4_microscaling_quantization_b200 import inputs

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


def noalloc_fn(fp4):
    from fp4_microscaling_quantization_b200 import _lib
    f = _lib.lib().fp4_gemm_decode_noalloc
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, i64, vp]
    f.restype = i32
    return f


@pytest.mark.parametrize("fmt,M,N,K", [(1, 16, 14336, 4096), (0, 4, 4096, 1024), (1, 1, 300, 512)])
def test_noalloc_matches_workspace_entry_point(fp4, fmt, M, N, K):
    import torch
    f = noalloc_fn(fp4)
    a, w = inputs.decode_linear(M, N, K, seed=M + N)
    A = fp4.quantize(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda(), fmt)
    W = fp4.quantize(torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).cuda(), fmt)
    ref = fp4.gemm(A, W, M, N, K, fmt, out_dtype=fp4.FP4_OUT_F32).cpu().numpy().astype(np.float64)
    # the GEMM tolerance: 1e-5 * sum_k |a_k||w_k| over the dequantized operands
    ah = fp4.dequantize(*A, fmt).cpu().numpy()
    wh = fp4.dequantize(*W, fmt).cpu().numpy()
    bound = np.abs(ah).astype(np.float64) @ np.abs(wh).astype(np.float64).T
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = f(A[0].data_ptr(), A[1].data_ptr(), A[2].data_ptr(), W[0].data_ptr(), W[1].data_ptr(),
               W[2].data_ptr(), M, N, K, fmt, fp4.FP4_OUT_F32, C.data_ptr(), N, stream)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        got = C.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= 1e-5 * bound), f"call {call} differs from fp4_gemm"


def test_noalloc_rejects_what_it_cannot_hold(fp4):
    f = noalloc_fn(fp4)
    import torch
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    p = z.data_ptr()
    # M above the decode range, and K not a multiple of 32: refused before any launch
    assert f(p, p, g.data_ptr(), p, p, g.data_ptr(), 17, 8, 256, 0, 0, p, 8, None) == 2
    assert f(p, p, g.data_ptr(), p, p, g.data_ptr(), 4, 8, 100, 0, 0, p, 8, None) == 2
    # Partials larger than the fixed array: many more tiles than SMs with two
    # K steps each, so the stream-K split cuts tiles and every CTA holds
    # several segments.  The size is settled on the host first, and every
    # buffer is allocated at full size, so the call could run safely even if
    # it were accepted.
    M, K, fmt = 16, 512, 0
    N = 128 * 600
    while fp4.gemm_workspace_size(M, N, K, fmt) <= 4 << 20:
        N *= 2
        assert N <= 128 * 600 * 16, "no decode shape needs more than the fixed array"
    qa = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.zeros((128 * K // 32,), dtype=torch.uint8, device="cuda")
    qw = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.zeros(((N + 127) // 128 * 128 * K // 32,), dtype=torch.uint8, device="cuda")
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rc = f(qa.data_ptr(), sa.data_ptr(), g.data_ptr(), qw.data_ptr(), sw.data_ptr(), g.data_ptr(), M, N, K, fmt,
           0, c.data_ptr(), N, None)
    torch.cuda.synchronize()
    assert rc == 2
