"""ctypes binding of libfp4.so (the C ABI in include/fp4.h).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of quantization and the GEMM runs in the library's
sm_100a kernels.  There is no fallback: if libfp4.so is missing or fails to
load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4.so")

FP4_MXFP4, FP4_NVFP4, FP4_MXFP4_16 = 0, 1, 2
FP4_ROUND_EVEN, FP4_ROUND_AWAY = 0, 1
FP4_MX_SCALE_CEIL, FP4_MX_SCALE_FLOOR = 0, 1
FP4_OUT_F32, FP4_OUT_BF16 = 0, 1
FP4_SCALE_ABSMAX, FP4_SCALE_MSE = 0, 1

STATUS = {
    0: "FP4_OK",
    1: "FP4_ERR_INVALID_ARG",
    2: "FP4_ERR_UNSUPPORTED",
    3: "FP4_ERR_ALIGNMENT",
    4: "FP4_ERR_CUDA",
    5: "FP4_ERR_TIMEOUT",
}

# every symbol the header declares, with (restype, argtypes)
_i64, _int, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "fp4_status_string": (ctypes.c_char_p, [_int]),
    "fp4_quantize_sizes": (_int, [_i64, _i64, _int, _int, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "fp4_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _vp, _vp, _vp, _vp, _vp]),
    "fp4_dequantize": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _int, _int, _int, _vp, _vp]),
    "fp4_gemm_workspace_size": (_int, [_i64, _i64, _i64, _int, ctypes.POINTER(_sz)]),
    "fp4_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _vp, _i64,
                        _vp, _sz, _vp]),
    "fp4_mx_to_nv_scales": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "fp4_quantize_residual": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fp4_dequantize_residual": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _int, _int, _vp, _vp]),
    "fp4_nv_refine_gscale_workspace_size": (_int, [_i64, _i64, _vp]),
    "fp4_nv_refine_gscale": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _int, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp]),
    "fp4_gemm_quantized": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp,
                                  _vp, _vp]),
    "fp4_check_device_status": (_int, [_vp]),
    "fp4_linear_workspace_size": (_int, [_i64, _i64, _i64, _int, ctypes.POINTER(_sz)]),
    "fp4_linear": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _i64, _int, _vp, _i64,
                          _vp, _sz, _vp]),
    "fp4_linear_residual": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _i64, _int, _vp, _i64,
                                   _vp]),
    "fp4_kernel_launches": (ctypes.c_uint64, []),
    "fp4_test_inject_stall": (_int, [_int, ctypes.c_uint64]),
}


class Fp4Opts(ctypes.Structure):
    _fields_ = [("round", ctypes.c_int), ("mx_scale_rule", ctypes.c_int), ("gscale_given", ctypes.c_int),
                ("scale_search", ctypes.c_int), ("weights_static", ctypes.c_int)]


class Fp4Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m fp4_microscaling_quantization_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(fn: str, code: int) -> None:
    if code != 0:
        raise Fp4Error(fn, code)
