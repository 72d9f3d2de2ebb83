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


# (fmt, M, N, K, uses the array): the last case takes whole tiles and needs no
# partial sums; the others cut tiles between CTAs (a few tiles split over many
# CTAs, or stream-K over more tiles than SMs), so their partials go through
# the library's array.
CASES = [(1, 1, 300, 512, True), (0, 16, 1000, 4096, True), (2, 4, 128 * 200, 512, True),
         (1, 16, 14336, 4096, False)]


def operands(fp4, fmt, M, N, K, seed):
    import torch
    a, w = inputs.decode_linear(M, N, K, seed=seed)
    A = fp4.quantize(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda(), fmt)
    W = fp4.quantize(torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).cuda(), fmt)
    return A, W


@pytest.mark.parametrize("fmt,M,N,K,uses_array", CASES)
def test_noalloc_matches_workspace_entry_point(fp4, fmt, M, N, K, uses_array):
    import torch
    f = noalloc_fn(fp4)
    assert (fp4.gemm_workspace_size(M, N, K, fmt) > 0) == uses_array
    A, W = operands(fp4, fmt, M, N, K, seed=M + N)
    # other operands of the same shape: a call with them leaves different
    # partial sums in the shared array, so a partial that a later call failed
    # to write would show up as a wrong result
    A2, W2 = operands(fp4, fmt, M, N, K, seed=M + N + 7)
    # the GEMM tolerance: 1e-5 * sum_k |a_k||w_k| over the dequantized operands
    ah = fp4.dequantize(*A, fmt).cpu().numpy()
    wh = fp4.dequantize(*W, fmt).cpu().numpy()
    bound = np.abs(ah).astype(np.float64) @ np.abs(wh).astype(np.float64).T
    stream = torch.cuda.current_stream().cuda_stream

    def call(Aop, Wop, out_dtype, C):
        return f(Aop[0].data_ptr(), Aop[1].data_ptr(), Aop[2].data_ptr(), Wop[0].data_ptr(), Wop[1].data_ptr(),
                 Wop[2].data_ptr(), M, N, K, fmt, out_dtype, C.data_ptr(), N, stream)

    for out_dtype, dt in ((fp4.FP4_OUT_F32, torch.float32), (fp4.FP4_OUT_BF16, torch.bfloat16)):
        ref = fp4.gemm(A, W, M, N, K, fmt, out_dtype=out_dtype).float().cpu().numpy().astype(np.float64)
        tol = 1e-5 * bound + (2.0 ** -8 * np.abs(ref) if out_dtype == fp4.FP4_OUT_BF16 else 0.0)
        dirty = torch.empty((M, N), dtype=dt, device="cuda")
        assert call(A2, W2, out_dtype, dirty) == 0
        for n in range(2):
            C = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
            rc = call(A, W, out_dtype, C)
            assert rc == 0, f"call {n}: status {rc}"
            torch.cuda.synchronize()
            got = C.float().cpu().numpy().astype(np.float64)
            assert np.all(np.abs(got - ref) <= tol), f"call {n} ({dt}) differs from fp4_gemm"


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
