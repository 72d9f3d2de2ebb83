"""CPU oracle for microscaling FP4 quantization and the W4A4 product.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
CUDA library (``fp4_microscaling_quantization_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``fp4_oracle.c`` (plain C, one IEEE fp32 operation at
a time, fp64 for the GEMM reference).  This module only builds that file and
marshals numpy arrays into it.

Parity status of each function (what pins it, see tests/test_oracle_pins.py):
  e2m1 encode/decode      pinned: page magnitude set, brute-force argmin over
                          every fp32 value (tests/test_oracle_exhaustive.py)
  e4m3 encode/decode      pinned: page bit patterns, torch float8_e4m3fn cast
  mx scale exponent       pinned: closed form from the exponent bits, worked
                          example, brute force over all 254 E8M0 scales
  fwht                    pinned: explicit Sylvester matrix product (scipy)
  quantize / dequantize   pinned: worked examples, power-of-two invariants,
                          Eq.(2) norm identity
  gemm reference          pinned: numpy fp64 matmul
  MXFP4 -> NVFP4 scales   pinned: dequantized elements unchanged (exact)
                          within 17 binades, E4M3 rounding past them,
                          closed-form s_g (tests/test_oracle_pins.py)
  sparse residual lane    pinned: FP4 stream equals the plain quantizer on the
                          zeroed values, bf16 RNE against torch, one-value
                          units exact, NMSE below the plain quantizer
  NVFP4 s_g refinement    pinned: one round = the absmax s_g with an
                          independently summed error, the second round's
                          least-squares step recomputed in numpy, errors
                          non-increasing, all-zero tensor
                          (tests/test_oracle_mse_pins.py)
  MSE block-scale search  pinned: hand-derived blocks, exhaustive numpy search
                          over every representable scale, nearest-element
                          property (tests/test_oracle_mse_pins.py)
  MXFP4 on 16-element     pinned: scale bytes by a brute-force search over the
  blocks (MXFP4_16)       E8M0 scales per 16-block, elements by brute-force
                          nearest grid point, every element's error at most
                          the 32-block MXFP4 error (the finer grid contains the
                          coarse one below the block max), equal to MXFP4
                          where a unit's halves share its exponent
                          (tests/test_oracle_mx16_pins.py)
  INT4 group baseline     pinned: every element at a nearest level of its
                          group's grid s*{-7..7}, s = amax/7, the group max at
                          +-7; Table 5's INT4 NMSE reproduced within 5 %
                          (tests/test_oracle_transfp4_pins.py)
  TransFP4 (rotation +    pinned: with the INT4 candidate off it equals the
  residual + NV/INT4      NVFP4 residual-lane round trip bit for bit; each
  choice per unit)        unit's choice has the smaller error; Table 5's
                          TransFP4 NMSE reproduced within 6 %
  NMSE vs the page's table   directional only for MXFP4 / NVFP4 / rotated
                          MXFP4 (the page's generator is unknown) (the page's generator is unknown)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MXFP4, NVFP4 = 0, 1
# MXFP4 elements and E8M0 scales on 16-element blocks (the C oracle's MXFP4
# with block 16); the tag matches the CUDA library's format code.
MXFP4_16 = 2
TIE_EVEN, TIE_AWAY = 0, 1
MX_CEIL, MX_FLOOR = 0, 1
SCALE_ABSMAX, SCALE_MSE = 0, 1


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c into liboracle.so beside it (gcc, OpenMP, no FMA
    contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "fp4_oracle.h"))
    ):
        cmd = [
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fexcess-precision=standard", "-fopenmp", "-fPIC", "-shared",
            "-o", _LIB + ".tmp", _SRC, "-lm",
        ]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        vp = ctypes.c_void_p
        L.fp4o_e2m1_encode.argtypes = [f32, i32]
        L.fp4o_e2m1_encode.restype = i32
        L.fp4o_e2m1_decode.argtypes = [i32]
        L.fp4o_e2m1_decode.restype = ctypes.c_double
        L.fp4o_e4m3_encode.argtypes = [f32]
        L.fp4o_e4m3_encode.restype = i32
        L.fp4o_e4m3_decode.argtypes = [i32]
        L.fp4o_e4m3_decode.restype = ctypes.c_double
        L.fp4o_e8m0_decode.argtypes = [i32]
        L.fp4o_e8m0_decode.restype = ctypes.c_double
        L.fp4o_mx_scale_exponent.argtypes = [f32, i32]
        L.fp4o_mx_scale_exponent.restype = i32
        L.fp4o_hadamard_ck.argtypes = [i32]
        L.fp4o_hadamard_ck.restype = f32
        L.fp4o_fwht.argtypes = [vp, i32]
        L.fp4o_fwht.restype = None
        L.fp4o_quantize.argtypes = [vp, i64, i64, i64, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp]
        L.fp4o_quantize.restype = i32
        L.fp4o_quantize_f32.argtypes = [vp, i64, i64, i64, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp]
        L.fp4o_quantize_f32.restype = i32
        L.fp4o_dequantize.argtypes = [vp, vp, f32, i64, i64, i32, i32, i32, vp]
        L.fp4o_dequantize.restype = i32
        L.fp4o_scales_to_atoms.argtypes = [vp, i64, i64, vp]
        L.fp4o_scales_from_atoms.argtypes = [vp, i64, i64, vp]
        L.fp4o_gemm_ref.argtypes = [vp, vp, i64, i64, i64, vp, vp]
        L.fp4o_mx_scales_to_nv.argtypes = [vp, i64, i64, vp, vp]
        L.fp4o_quantize_residual.argtypes = [vp, i64, i64, i64, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.fp4o_quantize_residual.restype = i32
        L.fp4o_dequantize_residual.argtypes = [vp, vp, f32, vp, i64, i64, i32, i32, i32, vp]
        L.fp4o_dequantize_residual.restype = i32
        L.fp4o_nv_refine_gscale.argtypes = [vp, i64, i64, i64, i32, i32, i32, vp, vp]
        L.fp4o_nv_refine_gscale.restype = i32
        L.fp4o_mx_scales_to_nv.restype = i32
        L.fp4o_int4_quantize_f32.argtypes = [vp, i64, i64, i32, vp, vp]
        L.fp4o_int4_quantize_f32.restype = i32
        L.fp4o_int4_dequantize.argtypes = [vp, vp, i64, i64, i32, vp]
        L.fp4o_int4_dequantize.restype = i32
        L.fp4o_transfp4_f32.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp]
        L.fp4o_transfp4_f32.restype = i32
        L.fp4o_num_threads.restype = i32
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def block_of(fmt: int) -> int:
    return 32 if fmt == MXFP4 else 16


def _cfmt(fmt: int) -> int:
    """The C oracle's format code: MXFP4_16 is MXFP4 with block 16."""
    return MXFP4 if fmt == MXFP4_16 else fmt


# ---- scalar codecs --------------------------------------------------------
def e2m1_encode(v: float, tie: int = TIE_EVEN) -> int:
    return lib().fp4o_e2m1_encode(float(v), tie)


def e2m1_decode(code: int) -> float:
    return lib().fp4o_e2m1_decode(int(code))


def e4m3_encode(t: float) -> int:
    return lib().fp4o_e4m3_encode(float(t))


def e4m3_decode(b: int) -> float:
    return lib().fp4o_e4m3_decode(int(b))


def e8m0_decode(b: int) -> float:
    return lib().fp4o_e8m0_decode(int(b))


def mx_scale_exponent(amax: float, rule: int = MX_CEIL) -> int:
    return lib().fp4o_mx_scale_exponent(float(amax), rule)


def hadamard_ck(k: int) -> np.float32:
    return np.float32(lib().fp4o_hadamard_ck(k))


def fwht(y: np.ndarray, k: int) -> np.ndarray:
    """Rotate every contiguous k-chunk of a 1-D fp32 array (returns a copy)."""
    y = np.ascontiguousarray(y, dtype=np.float32).copy()
    assert y.size % k == 0
    for c in range(0, y.size, k):
        chunk = np.ascontiguousarray(y[c:c + k])
        lib().fp4o_fwht(_ptr(chunk), k)
        y[c:c + k] = chunk
    return y


# ---- tensors ----------------------------------------------------------------
def quantize(x_bf16: np.ndarray, fmt: int, hadamard_k: int = 0, tie: int = TIE_EVEN,
             mx_rule: int = MX_CEIL, gscale: float | None = None, search: int = SCALE_ABSMAX):
    """x_bf16: (rows, cols) uint16 bf16 bit patterns.  search: SCALE_ABSMAX
    or SCALE_MSE (block scales by the MSE search; mx_rule is then unused).

    Returns (q, s_logical, s_g): q (rows, cols/2) uint8 packed nibbles,
    s_logical (rows, cols/block) uint8, s_g the NVFP4 tensor scale (1.0 for MX).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    block = block_of(fmt)
    q = np.zeros((rows, cols // 2), np.uint8)
    s = np.zeros((rows, cols // block), np.uint8)
    g = np.array([gscale if gscale is not None else 0.0], np.float32)
    rc = lib().fp4o_quantize(_ptr(x), rows, cols, cols, _cfmt(fmt), block, hadamard_k, tie,
                             mx_rule, search, int(gscale is not None), _ptr(g), _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("oracle quantize: invalid arguments")
    return q, s, (float(g[0]) if fmt == NVFP4 else 1.0)


def quantize_f32(x: np.ndarray, fmt: int, hadamard_k: int = 0, tie: int = TIE_EVEN,
                 mx_rule: int = MX_CEIL, gscale: float | None = None, search: int = SCALE_ABSMAX):
    """quantize() for fp32 elements (rows, cols): same outputs."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    block = block_of(fmt)
    q = np.zeros((rows, cols // 2), np.uint8)
    s = np.zeros((rows, cols // block), np.uint8)
    g = np.array([gscale if gscale is not None else 0.0], np.float32)
    rc = lib().fp4o_quantize_f32(_ptr(x), rows, cols, cols, _cfmt(fmt), block, hadamard_k, tie,
                                 mx_rule, search, int(gscale is not None), _ptr(g), _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("oracle quantize: invalid arguments")
    return q, s, (float(g[0]) if fmt == NVFP4 else 1.0)


def dequantize(q: np.ndarray, s_logical: np.ndarray, gscale: float, fmt: int,
               hadamard_k: int = 0) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s_logical, dtype=np.uint8)
    rows, half = q.shape
    cols = half * 2
    out = np.zeros((rows, cols), np.float32)
    rc = lib().fp4o_dequantize(_ptr(q), _ptr(s), float(gscale), rows, cols, _cfmt(fmt),
                               block_of(fmt), hadamard_k, _ptr(out))
    if rc != 0:
        raise ValueError("oracle dequantize: invalid arguments")
    return out


def scales_to_atoms(s_logical: np.ndarray) -> np.ndarray:
    s = np.ascontiguousarray(s_logical, dtype=np.uint8)
    rows, nkb = s.shape
    out = np.zeros(((rows + 127) // 128 * 128) * ((nkb + 3) // 4 * 4), np.uint8)
    lib().fp4o_scales_to_atoms(_ptr(s), rows, nkb, _ptr(out))
    return out


def scales_from_atoms(s_atoms: np.ndarray, rows: int, nkb: int) -> np.ndarray:
    a = np.ascontiguousarray(s_atoms, dtype=np.uint8)
    out = np.zeros((rows, nkb), np.uint8)
    lib().fp4o_scales_from_atoms(_ptr(a), rows, nkb, _ptr(out))
    return out


def quantize_residual(x_bf16: np.ndarray, fmt: int, hadamard_k: int = 0, tie: int = TIE_EVEN,
                      mx_rule: int = MX_CEIL, gscale: float | None = None):
    """quantize() with the sparse residual lane (TransFP4 Eq.(3), one value
    per 32): returns (q, s_logical, s_g, res), res (rows, cols/32) uint32
    words = bf16 bits | index << 16."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    block = block_of(fmt)
    q = np.zeros((rows, cols // 2), np.uint8)
    s = np.zeros((rows, cols // block), np.uint8)
    res = np.zeros((rows, cols // 32), np.uint32)
    g = np.array([gscale if gscale is not None else 0.0], np.float32)
    rc = lib().fp4o_quantize_residual(_ptr(x), rows, cols, cols, _cfmt(fmt), block, hadamard_k, tie, mx_rule,
                                      int(gscale is not None), _ptr(g), _ptr(q), _ptr(s), _ptr(res))
    if rc != 0:
        raise ValueError("oracle quantize_residual: invalid arguments")
    return q, s, (float(g[0]) if fmt == NVFP4 else 1.0), res


def dequantize_residual(q, s_logical, gscale, res, fmt, hadamard_k: int = 0):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s_logical, dtype=np.uint8)
    r = np.ascontiguousarray(res, dtype=np.uint32)
    rows, half = q.shape
    cols = half * 2
    out = np.zeros((rows, cols), np.float32)
    if lib().fp4o_dequantize_residual(_ptr(q), _ptr(s), float(gscale), _ptr(r), rows, cols, _cfmt(fmt),
                                      block_of(fmt), hadamard_k, _ptr(out)) != 0:
        raise ValueError("oracle dequantize_residual: invalid arguments")
    return out


def nv_refine_gscale(x_bf16: np.ndarray, hadamard_k: int = 0, tie: int = TIE_EVEN, rounds: int = 4):
    """Alternating refinement of the NVFP4 tensor scale: (s_g, its squared
    error) after `rounds` MSE-group / least-squares-global rounds."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, cols = x.shape
    g = np.zeros(1, np.float32)
    e = np.zeros(1, np.float64)
    if lib().fp4o_nv_refine_gscale(_ptr(x), rows, cols, cols, hadamard_k, tie, rounds, _ptr(g), _ptr(e)) != 0:
        raise ValueError("oracle nv_refine_gscale: invalid arguments")
    return float(g[0]), float(e[0])


def mx_scales_to_nv(s_mx_logical: np.ndarray):
    """MXFP4 scales (rows, nkb) -> (NVFP4 scales (rows, 2 nkb), s_g) with the
    same dequantized elements (late binding of an MXFP4 weight to NVFP4)."""
    s = np.ascontiguousarray(s_mx_logical, dtype=np.uint8)
    rows, nkb = s.shape
    out = np.zeros((rows, 2 * nkb), np.uint8)
    g = np.zeros(1, np.float32)
    if lib().fp4o_mx_scales_to_nv(_ptr(s), rows, nkb, _ptr(out), _ptr(g)) != 0:
        raise ValueError("oracle mx_scales_to_nv: invalid arguments")
    return out, float(g[0])


def int4_quantize(x: np.ndarray, group: int = 32):
    """INT4 group quantization of fp32 rows (Table 5's INT4 baseline):
    returns (q int8 (rows, cols), scales fp32 (rows, cols/group))."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.int8)
    s = np.zeros((rows, cols // group if group else 0), np.float32)
    if lib().fp4o_int4_quantize_f32(_ptr(x), rows, cols, group, _ptr(q), _ptr(s)) != 0:
        raise ValueError("oracle int4_quantize: invalid arguments")
    return q, s


def int4_dequantize(q: np.ndarray, s: np.ndarray, group: int = 32) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    rows, cols = q.shape
    out = np.zeros((rows, cols), np.float32)
    if lib().fp4o_int4_dequantize(_ptr(q), _ptr(s), rows, cols, group, _ptr(out)) != 0:
        raise ValueError("oracle int4_dequantize: invalid arguments")
    return out


def transfp4(x: np.ndarray, hadamard_k: int = 32, tie: int = TIE_EVEN, allow_int4: bool = True):
    """The TransFP4 method of the page's Table 5 on fp32 rows (rotation,
    residual lane, per-unit NVFP4 / INT4 choice): returns (x_hat fp32
    (rows, cols), choice uint8 (rows, cols/32), 1 = INT4)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    out = np.zeros((rows, cols), np.float32)
    choice = np.zeros((rows, cols // 32), np.uint8)
    if lib().fp4o_transfp4_f32(_ptr(x), rows, cols, hadamard_k, tie, int(bool(allow_int4)), _ptr(out),
                               _ptr(choice)) != 0:
        raise ValueError("oracle transfp4: invalid arguments")
    return out, choice


def gemm_ref(a_hat: np.ndarray, w_hat: np.ndarray):
    """fp64 C = A W^T and the per-element bound sum_k |a||w|."""
    a = np.ascontiguousarray(a_hat, dtype=np.float32)
    w = np.ascontiguousarray(w_hat, dtype=np.float32)
    M, K = a.shape
    N, K2 = w.shape
    assert K == K2
    c = np.zeros((M, N), np.float64)
    b = np.zeros((M, N), np.float64)
    lib().fp4o_gemm_ref(_ptr(a), _ptr(w), M, N, K, _ptr(c), _ptr(b))
    return c, b


def num_threads() -> int:
    return lib().fp4o_num_threads()


def nmse(x: np.ndarray, x_hat: np.ndarray) -> float:
    """||x - x_hat||^2 / ||x||^2 ("Portable FP4 quantization", §3.2)."""
    x = np.asarray(x, np.float64)
    d = x - np.asarray(x_hat, np.float64)
    return float(np.sum(d * d) / np.sum(x * x))
