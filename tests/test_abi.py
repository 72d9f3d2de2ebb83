"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
and rejects invalid calls on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

from fp4_microscaling_quantization_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fp4_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert "fp4_quantize" in names and "fp4_gemm" in names
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(_lib.SIGNATURES) <= names


def test_status_strings(L):
    for code in range(6):
        assert L.fp4_status_string(code).startswith(b"FP4_")


def test_quantize_sizes(L):
    q, s = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.fp4_quantize_sizes(200, 320, 0, 32, ctypes.byref(q), ctypes.byref(s)) == 0
    assert q.value == 200 * 160 and s.value == 256 * 12
    assert L.fp4_quantize_sizes(200, 320, 1, 16, ctypes.byref(q), ctypes.byref(s)) == 0
    assert s.value == 256 * 20
    # MXFP4 with block 16 is MXFP4_16: 16-element blocks, E8M0 scales
    assert L.fp4_quantize_sizes(200, 320, 0, 16, ctypes.byref(q), ctypes.byref(s)) == 0
    assert q.value == 200 * 160 and s.value == 256 * 20
    assert L.fp4_quantize_sizes(200, 320, 2, 16, ctypes.byref(q), ctypes.byref(s)) == 0
    assert s.value == 256 * 20
    assert L.fp4_quantize_sizes(4, 64, 2, 32, ctypes.byref(q), ctypes.byref(s)) == 2  # MXFP4_16 is 16
    assert L.fp4_quantize_sizes(4, 64, 0, 8, ctypes.byref(q), ctypes.byref(s)) == 2
    assert L.fp4_quantize_sizes(-1, 64, 0, 32, ctypes.byref(q), ctypes.byref(s)) == 1
    # byte counts that do not fit in 63 bits are rejected, not wrapped
    assert L.fp4_quantize_sizes(1 << 40, 1 << 30, 0, 32, ctypes.byref(q), ctypes.byref(s)) == 1
    assert L.fp4_quantize_sizes(1 << 31, 1 << 32, 1, 16, ctypes.byref(q), ctypes.byref(s)) == 0
    assert q.value == (1 << 31) * (1 << 31) and s.value == (1 << 31) * (1 << 28)


FAKE = 0x10000  # an aligned pointer value never dereferenced: validation fails first


@pytest.mark.parametrize("args,code", [
    (dict(rows=-1), 1),
    (dict(fmt=0, block=8), 2),
    (dict(fmt=1, block=32), 2),
    (dict(fmt=2, block=32), 2),
    (dict(fmt=3, block=16), 2),
    (dict(hadamard_k=8), 2),
    (dict(cols=48), 2),
    (dict(cols=64, hadamard_k=128), 2),
    (dict(ld=16), 1),
    (dict(x=FAKE + 8), 3),
    (dict(ld=68), 3),
    (dict(q=FAKE + 4), 3),
    (dict(fmt=1, block=16, g=None), 1),
    (dict(x=None), 1),
])
def test_quantize_rejects_on_host(L, args, code):
    a = dict(x=FAKE, rows=4, cols=64, ld=64, fmt=0, block=32, hadamard_k=0, q=FAKE, s=FAKE, g=FAKE)
    a.update(args)
    rc = L.fp4_quantize(a["x"], a["rows"], a["cols"], a["ld"], a["fmt"], a["block"], a["hadamard_k"],
                        None, a["q"], a["s"], a["g"], None)
    assert rc == code


def test_bad_opts_rejected(L):
    o = _lib.Fp4Opts(7, 0, 0)
    assert L.fp4_quantize(FAKE, 4, 64, 64, 0, 32, 0, ctypes.byref(o), FAKE, FAKE, FAKE, None) == 1
    o = _lib.Fp4Opts(0, 3, 0)
    assert L.fp4_quantize(FAKE, 4, 64, 64, 0, 32, 0, ctypes.byref(o), FAKE, FAKE, FAKE, None) == 1
    o = _lib.Fp4Opts(0, 0, 0, 2)  # no such scale method
    assert L.fp4_quantize(FAKE, 4, 64, 64, 0, 32, 0, ctypes.byref(o), FAKE, FAKE, FAKE, None) == 1


def test_mse_scales_only_in_quantize(L):
    o = _lib.Fp4Opts(0, 0, 0, _lib.FP4_SCALE_MSE)
    F = FAKE
    assert L.fp4_linear(F, 4, 256, 256, 0, 0, ctypes.byref(o), None, F, F, F, 8, 1, F, 8, F, 1 << 20, None) == 2
    assert L.fp4_gemm_quantized(F, F, F, F, F, F, 256, 256, 256, 0, 0, ctypes.byref(o), None, F, F, None) == 2


def test_dequantize_rejects_on_host(L):
    assert L.fp4_dequantize(FAKE, FAKE, FAKE, 4, 64, 0, 32, 0, 9, FAKE, None) == 1
    assert L.fp4_dequantize(FAKE, FAKE, None, 4, 64, 1, 16, 0, 0, FAKE, None) == 1
    assert L.fp4_dequantize(FAKE + 1, FAKE, FAKE, 4, 64, 0, 32, 0, 0, FAKE, None) == 3
    assert L.fp4_dequantize(FAKE, FAKE, FAKE, 4, 48, 0, 32, 0, 0, FAKE, None) == 2


def test_gemm_rejects_on_host(L):
    g = L.fp4_gemm
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 100, 0, 1, FAKE, 8, None, 0, None) == 2  # K % 32
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 256, 0, 1, FAKE, 4, None, 0, None) == 1  # ldc < N
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 256, 5, 1, FAKE, 8, None, 0, None) == 2
    assert g(None, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 256, 0, 1, FAKE, 8, None, 0, None) == 1
    assert g(FAKE, FAKE, None, FAKE, FAKE, FAKE, 4, 8, 256, 1, 1, FAKE, 8, None, 0, None) == 1
    assert g(FAKE + 2, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 256, 0, 1, FAKE, 8, None, 0, None) == 3


def test_sizes_beyond_2_30_rejected(L):
    b = ctypes.c_size_t()
    assert L.fp4_gemm_workspace_size(4, (1 << 30) + 1, 256, 0, ctypes.byref(b)) == 2
    assert L.fp4_linear_workspace_size(4, 256, (1 << 31), 1, ctypes.byref(b)) == 2
    assert L.fp4_linear_workspace_size(4, 256, 1024, 2, ctypes.byref(b)) == 0 and b.value > 0
    F = FAKE
    assert L.fp4_linear(F, 4, 1 << 31, 1 << 31, 0, 0, None, None, F, F, F, 8, 1, F, 8, F, 1 << 20, None) == 2


def test_gemm_quantized_rejects_on_host(L):
    g = L.fp4_gemm_quantized
    F = FAKE
    assert g(F, F, F, F, F, F, 16, 256, 256, 0, 0, None, None, F, F, None) == 2      # M <= 16: decode shapes
    assert g(F, F, F, F, F, F, 256, 192, 256, 0, 0, None, None, F, F, None) == 2     # N % 128
    assert g(F, F, F, F, F, F, 256, 256, 112, 0, 0, None, None, F, F, None) == 2     # K % 32
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 3, None, None, F, F, None) == 2     # output format
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 2, None, None, F, F, None) == 2     # no MXFP4_16 output
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 1, None, None, F, F, None) == 1     # NVFP4 out needs gC
    assert g(F, F, None, F, F, F, 256, 256, 256, 1, 0, None, None, F, F, None) == 1  # NVFP4 in needs gA
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 0, None, None, None, F, None) == 1  # Cq
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 0, None, None, F + 4, F, None) == 3
    o = _lib.Fp4Opts(7, 0, 0)
    assert g(F, F, F, F, F, F, 256, 256, 256, 0, 0, ctypes.byref(o), None, F, F, None) == 1


def test_residual_rejects_on_host(L):
    F = FAKE
    o = _lib.Fp4Opts(0, 0, 0, _lib.FP4_SCALE_MSE, 0)
    assert L.fp4_quantize_residual(F, 4, 64, 64, 0, 32, 0, ctypes.byref(o), F, F, F, F, None) == 2
    assert L.fp4_quantize_residual(F, 4, 64, 64, 0, 32, 0, None, F, F, F, None, None) == 1  # res
    assert L.fp4_quantize_residual(F, 4, 64, 64, 0, 32, 0, None, F, F, F, F + 2, None) == 3
    assert L.fp4_dequantize_residual(F, F, F, None, 4, 64, 0, 32, 0, 0, F, None) == 1
    assert L.fp4_dequantize_residual(F, F, F, F, 4, 48, 0, 32, 0, 0, F, None) == 2


def test_refine_rejects_on_host(L):
    F = FAKE
    g = L.fp4_nv_refine_gscale
    assert g(F, 4, 64, 64, 0, None, 0, F, F, F, 1 << 20, F, None) == 1       # rounds < 1
    assert g(F, 4, 64, 64, 0, None, 65, F, F, F, 1 << 20, F, None) == 1      # rounds > 64
    assert g(F, 4, 48, 64, 0, None, 2, F, F, F, 1 << 20, F, None) == 2       # cols % 32
    assert g(F, 4, 64, 64, 0, None, 2, F, F, F, 16, F, None) == 1            # workspace too small
    assert g(F, 4, 64, 64, 0, None, 2, F, F, F + 16, 1 << 20, F, None) == 3  # workspace alignment


def test_empty_mx_is_noop(L):
    assert L.fp4_quantize(None, 0, 64, 64, 0, 32, 0, None, None, None, None, None) == 0
    assert L.fp4_dequantize(None, None, None, 0, 64, 0, 32, 0, 0, None, None) == 0


def test_binding_refuses_host_tensors():
    """The Python binding passes raw device pointers: a host tensor (or a short
    buffer) is refused before anything reaches the library."""
    import torch
    import fp4_microscaling_quantization_b200 as fp4
    M, N, K = 4, 256, 512
    qa = torch.zeros((M, K // 2), dtype=torch.uint8)
    sa = torch.zeros((fp4.quantize_sizes(M, K, 0)[1],), dtype=torch.uint8)
    qw = torch.zeros((N, K // 2), dtype=torch.uint8)
    sw = torch.zeros((fp4.quantize_sizes(N, K, 0)[1],), dtype=torch.uint8)
    g = torch.ones((1,), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp4.gemm((qa, sa, g), (qw, sw, g), M, N, K, 0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp4.gemm_quantized((qa, sa, g), (qw, sw, g), M, N, K, 0, 0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp4.dequantize(qa, sa, g, 0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fp4.linear(torch.zeros((M, K), dtype=torch.bfloat16), (qw, sw, g), 0)
    with pytest.raises(ValueError):
        fp4.quantize(torch.zeros((M, K), dtype=torch.bfloat16), 0)
    # shapes the library rejects are refused while sizing the operands
    with pytest.raises(fp4.Fp4Error):
        fp4.gemm((qa, sa, g), (qw, sw, g), M, N, 100, 0)
