"""B200 (sm_100a) microscaling FP4: MXFP4 / NVFP4 quantization with a fused
block-diagonal Hadamard rotation, and the block-scaled W4A4 GEMM.

Python front end of the C ABI in include/fp4.h.  Tensors are torch CUDA
tensors (device memory and the current stream come from torch); all
arithmetic runs in libfp4.so.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (FP4_MX_SCALE_CEIL, FP4_MX_SCALE_FLOOR, FP4_MXFP4, FP4_MXFP4_16, FP4_NVFP4, FP4_OUT_BF16,
                   FP4_OUT_F32, FP4_ROUND_AWAY, FP4_ROUND_EVEN, FP4_SCALE_ABSMAX, FP4_SCALE_MSE, Fp4Error)

__all__ = [
    "quantize", "dequantize", "gemm", "gemm_quantized", "linear", "linear_residual", "linear_workspace_size",
    "quantize_sizes",
    "gemm_workspace_size", "check_device_status", "kernel_launches",
    "FP4_MXFP4", "FP4_NVFP4", "FP4_MXFP4_16", "FP4_ROUND_EVEN", "FP4_ROUND_AWAY", "FP4_MX_SCALE_CEIL",
    "FP4_MX_SCALE_FLOOR", "FP4_OUT_F32", "FP4_OUT_BF16", "FP4_SCALE_ABSMAX", "FP4_SCALE_MSE",
    "Fp4Error", "block_of",
]


def block_of(fmt: int) -> int:
    """Elements per block: 32 for MXFP4, 16 for NVFP4 and MXFP4_16."""
    return 32 if fmt == FP4_MXFP4 else 16


def _fmt(fmt) -> int:
    if isinstance(fmt, str):
        return {"mxfp4": FP4_MXFP4, "nvfp4": FP4_NVFP4, "mxfp4_16": FP4_MXFP4_16}[fmt.lower()]
    return int(fmt)


def _stream_handle(torch, device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _run(name: str, device, *args) -> None:
    """Calls entry point `name` of the library with `device` current.  The
    library launches on the current device and takes the SM count and the
    scratch it uses from it, so that must be the device whose memory and
    stream the call is given."""
    import torch

    with torch.cuda.device(device):
        _lib.check(name, getattr(_lib.lib(), name)(*args))


def _dev(t, name: str, device, dtype=None, min_bytes: int = 0, contiguous: bool = True):
    """Checks a tensor whose device pointer goes to the library: a CUDA tensor
    on `device`, of `dtype`, contiguous, holding at least `min_bytes` bytes.
    The library sees only the pointer, so a host tensor or a short buffer
    would otherwise be read or written out of bounds on the device."""
    import torch

    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, {min_bytes} needed")
    return t


def _operand(t3, rows: int, cols: int, fmt: int, name: str, device):
    """A quantized operand (q, s, g) of a rows x cols tensor in format fmt."""
    import torch

    q, s, g = t3
    qb, sb = quantize_sizes(rows, cols, fmt)
    _dev(q, name + " elements", device, torch.uint8, qb)
    _dev(s, name + " scales", device, torch.uint8, sb)
    _dev(g, name + " tensor scale", device, torch.float32, 4)
    return q, s, g


def _out2d(out, rows: int, cols: int, dtype, name: str, device):
    """A row-major output of at least rows x cols (its row stride is passed on)."""
    _dev(out, name, device, dtype, contiguous=False)
    if out.dim() != 2 or out.shape[0] < rows or out.shape[1] < cols or (out.numel() and out.stride(1) != 1):
        raise ValueError(f"{name} must be a 2-D tensor of at least {rows} x {cols}, contiguous along its rows")
    return out


def quantize_sizes(rows: int, cols: int, fmt) -> tuple[int, int]:
    fmt = _fmt(fmt)
    qb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _lib.check("fp4_quantize_sizes",
               _lib.lib().fp4_quantize_sizes(rows, cols, fmt, block_of(fmt), ctypes.byref(qb), ctypes.byref(sb)))
    return qb.value, sb.value


def quantize(x, fmt, hadamard_k: int = 0, round: int = FP4_ROUND_EVEN,
             mx_scale_rule: int = FP4_MX_SCALE_CEIL, gscale=None, out=None,
             scale_search: int = FP4_SCALE_ABSMAX):
    """Quantize a 2-D bf16 CUDA tensor along its last axis.

    Returns (q, s, g): q uint8 (rows, cols/2) packed nibbles, s uint8 scales in
    the tensor-core tile layout, g a 1-element fp32 tensor holding s_g (NVFP4;
    for MXFP4 a tensor holding 1).  If ``gscale`` is given (NVFP4) it is used
    as s_g instead of computing it.  ``out`` = (q, s, g) reuses buffers.
    ``scale_search`` = FP4_SCALE_MSE picks each block scale by the MSE search.
    """
    import torch

    fmt = _fmt(fmt)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bf16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must be contiguous along its last axis")
    rows, cols = x.shape
    qb, sb = quantize_sizes(rows, cols, fmt)
    if out is None:
        q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
        s = torch.empty((sb,), dtype=torch.uint8, device=x.device)
        g = torch.ones((1,), dtype=torch.float32, device=x.device)
    else:
        q, s, g = out
        _dev(q, "q", x.device, torch.uint8, qb)
        _dev(s, "s", x.device, torch.uint8, sb)
        _dev(g, "g", x.device, torch.float32, 4)
    given = gscale is not None
    if given:
        g.copy_(gscale.reshape(1).to(torch.float32))
    opts = _lib.Fp4Opts(int(round), int(mx_scale_rule), int(given), int(scale_search))
    gp = g.data_ptr() if fmt == FP4_NVFP4 else None
    _run("fp4_quantize", x.device,
        x.data_ptr(), rows, cols, x.stride(0), fmt, block_of(fmt), int(hadamard_k), ctypes.byref(opts),
        q.data_ptr(), s.data_ptr(), gp, _stream_handle(torch, x.device))
    return q, s, g


def dequantize(q, s, g, fmt, hadamard_k: int = 0, out_dtype: int = FP4_OUT_F32, out=None):
    """Inverse of :func:`quantize`; returns a (rows, cols) fp32 or bf16 tensor."""
    import torch

    fmt = _fmt(fmt)
    rows, half = q.shape
    cols = half * 2
    dt = torch.float32 if out_dtype == FP4_OUT_F32 else torch.bfloat16
    _operand((q, s, g), rows, cols, fmt, "x", q.device)
    if out is None:
        out = torch.empty((rows, cols), dtype=dt, device=q.device)
    _dev(out, "out", q.device, dt, rows * cols * (4 if dt == torch.float32 else 2))
    gp = g.data_ptr() if fmt == FP4_NVFP4 else None
    _run("fp4_dequantize", q.device,
        q.data_ptr(), s.data_ptr(), gp, rows, cols, fmt, block_of(fmt), int(hadamard_k), int(out_dtype),
        out.data_ptr(), _stream_handle(torch, q.device))
    return out


def gemm_workspace_size(M: int, N: int, K: int, fmt) -> int:
    b = ctypes.c_size_t()
    _lib.check("fp4_gemm_workspace_size",
               _lib.lib().fp4_gemm_workspace_size(M, N, K, _fmt(fmt), ctypes.byref(b)))
    return b.value


def gemm(a, w, M: int, N: int, K: int, fmt, out_dtype: int = FP4_OUT_BF16, out=None, workspace=None):
    """C = A W^T from quantized operands a = (Aq, As, gA), w = (Wq, Ws, gW)."""
    import torch

    fmt = _fmt(fmt)
    dev = a[0].device
    Aq, As, gA = _operand(a, M, K, fmt, "A", dev)
    Wq, Ws, gW = _operand(w, N, K, fmt, "W", dev)
    dt = torch.float32 if out_dtype == FP4_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=Aq.device)
    _out2d(out, M, N, dt, "out", dev)
    need = gemm_workspace_size(M, N, K, fmt)
    if need and workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=Aq.device)
    if workspace is not None:
        _dev(workspace, "workspace", dev, torch.uint8)
    wp = workspace.data_ptr() if workspace is not None else None
    wb = workspace.numel() if workspace is not None else 0
    _run("fp4_gemm", Aq.device,
        Aq.data_ptr(), As.data_ptr(), gA.data_ptr(), Wq.data_ptr(), Ws.data_ptr(), gW.data_ptr(),
        M, N, K, fmt, int(out_dtype), out.data_ptr(), out.stride(0), wp, wb,
        _stream_handle(torch, Aq.device))
    return out


def gemm_quantized(a, w, M: int, N: int, K: int, fmt, out_fmt, gscale=None, round: int = FP4_ROUND_EVEN,
                   mx_scale_rule: int = FP4_MX_SCALE_CEIL, out=None):
    """C = A W^T quantized along N for the next layer, in the GEMM's epilogue.

    a = (Aq, As, gA), w = (Wq, Ws, gW) as for :func:`gemm`.  Returns
    (Cq, Cs, gC) like :func:`quantize`: Cq (M, N/2) packed nibbles, Cs the
    tile-layout scales, gC the NVFP4 tensor scale of C, which must be given
    (``gscale``) for an NVFP4 output.
    """
    import torch

    fmt, out_fmt = _fmt(fmt), _fmt(out_fmt)
    dev = a[0].device
    Aq, As, gA = _operand(a, M, K, fmt, "A", dev)
    Wq, Ws, gW = _operand(w, N, K, fmt, "W", dev)
    qb, sb = quantize_sizes(M, N, out_fmt)
    if out is None:
        Cq = torch.empty((M, N // 2), dtype=torch.uint8, device=Aq.device)
        Cs = torch.empty((sb,), dtype=torch.uint8, device=Aq.device)
        gC = torch.ones((1,), dtype=torch.float32, device=Aq.device)
    else:
        Cq, Cs, gC = out
        _operand(out, M, N, out_fmt, "C", dev)
    if gscale is not None:
        gC.copy_(gscale.reshape(1).to(torch.float32))
    opts = _lib.Fp4Opts(int(round), int(mx_scale_rule), int(gscale is not None))
    _run("fp4_gemm_quantized", Aq.device,
        Aq.data_ptr(), As.data_ptr(), gA.data_ptr(), Wq.data_ptr(), Ws.data_ptr(), gW.data_ptr(),
        M, N, K, fmt, out_fmt, ctypes.byref(opts), gC.data_ptr() if out_fmt == FP4_NVFP4 else None,
        Cq.data_ptr(), Cs.data_ptr(), _stream_handle(torch, Aq.device))
    return Cq, Cs, gC


def quantize_residual(x, fmt, hadamard_k: int = 0, round: int = FP4_ROUND_EVEN,
                      mx_scale_rule: int = FP4_MX_SCALE_CEIL, gscale=None):
    """:func:`quantize` with the sparse residual lane (TransFP4 Eq.(3), one
    value per 32): returns (q, s, g, res), res (rows, cols/32) int32 words =
    bf16 bits | index << 16."""
    import torch

    fmt = _fmt(fmt)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 CUDA tensor, contiguous along its last axis")
    rows, cols = x.shape
    _, sb = quantize_sizes(rows, cols, fmt)
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    s = torch.empty((sb,), dtype=torch.uint8, device=x.device)
    g = torch.ones((1,), dtype=torch.float32, device=x.device)
    res = torch.empty((rows, cols // 32), dtype=torch.int32, device=x.device)
    given = gscale is not None
    if given:
        g.copy_(gscale.reshape(1).to(torch.float32))
    opts = _lib.Fp4Opts(int(round), int(mx_scale_rule), int(given), 0, 0)
    _run("fp4_quantize_residual", x.device,
        x.data_ptr(), rows, cols, x.stride(0), fmt, block_of(fmt), int(hadamard_k), ctypes.byref(opts),
        q.data_ptr(), s.data_ptr(), g.data_ptr() if fmt == FP4_NVFP4 else None, res.data_ptr(),
        _stream_handle(torch, x.device))
    return q, s, g, res


def dequantize_residual(q, s, g, res, fmt, hadamard_k: int = 0, out_dtype: int = FP4_OUT_F32):
    """Inverse of :func:`quantize_residual`."""
    import torch

    fmt = _fmt(fmt)
    rows, cols = q.shape[0], q.shape[1] * 2
    _operand((q, s, g), rows, cols, fmt, "x", q.device)
    _dev(res, "res", q.device, None, rows * (cols // 32) * 4)
    out = torch.empty((rows, cols), dtype=torch.float32 if out_dtype == FP4_OUT_F32 else torch.bfloat16,
                      device=q.device)
    _run("fp4_dequantize_residual", q.device,
        q.data_ptr(), s.data_ptr(), g.data_ptr() if fmt == FP4_NVFP4 else None, res.data_ptr(), rows, cols, fmt,
        block_of(fmt), int(hadamard_k), int(out_dtype), out.data_ptr(), _stream_handle(torch, q.device))
    return out


def nv_refine_gscale(x, hadamard_k: int = 0, rounds: int = 4, round: int = FP4_ROUND_EVEN):
    """The NVFP4 tensor scale of x refined by alternating MSE group steps and
    least-squares global steps (see fp4_nv_refine_gscale); returns a
    1-element fp32 tensor for ``quantize(..., gscale=...,
    scale_search=FP4_SCALE_MSE)``."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 CUDA tensor, contiguous along its last axis")
    rows, cols = x.shape
    qb, sb = quantize_sizes(rows, cols, FP4_NVFP4)
    q = torch.empty((max(qb, 16),), dtype=torch.uint8, device=x.device)
    s = torch.empty((max(sb, 16),), dtype=torch.uint8, device=x.device)
    nb = ctypes.c_size_t()
    _lib.check("fp4_nv_refine_gscale_workspace_size",
               _lib.lib().fp4_nv_refine_gscale_workspace_size(rows, cols, ctypes.byref(nb)))
    ws = torch.empty((nb.value,), dtype=torch.uint8, device=x.device)
    g = torch.empty((1,), dtype=torch.float32, device=x.device)
    opts = _lib.Fp4Opts(int(round), 0, 0, 0, 0)
    _run("fp4_nv_refine_gscale", x.device,
        x.data_ptr(), rows, cols, x.stride(0), int(hadamard_k), ctypes.byref(opts), int(rounds), q.data_ptr(),
        s.data_ptr(), ws.data_ptr(), nb.value, g.data_ptr(), _stream_handle(torch, x.device))
    return g


def mx_to_nv(w):
    """An MXFP4 tensor w = (q, s, g) in the NVFP4 scale form (q, s_nv, s_g)
    with the same dequantized elements (see fp4_mx_to_nv_scales); q is shared."""
    import torch

    q, s, _ = w
    rows, cols = q.shape[0], q.shape[1] * 2
    _dev(s, "MXFP4 scales", q.device, torch.uint8, quantize_sizes(rows, cols, FP4_MXFP4)[1])
    _, sb = quantize_sizes(rows, cols, FP4_NVFP4)
    s_nv = torch.empty((sb,), dtype=torch.uint8, device=q.device)
    g = torch.empty((1,), dtype=torch.float32, device=q.device)
    _run("fp4_mx_to_nv_scales", q.device,
        s.data_ptr(), rows, cols, s_nv.data_ptr(), g.data_ptr(), _stream_handle(torch, q.device))
    return q, s_nv, g


def linear_workspace_size(M: int, N: int, K: int, fmt) -> int:
    b = ctypes.c_size_t()
    _lib.check("fp4_linear_workspace_size",
               _lib.lib().fp4_linear_workspace_size(M, N, K, _fmt(fmt), ctypes.byref(b)))
    return b.value


def linear(x, w, fmt, hadamard_k: int = 0, out_dtype: int = FP4_OUT_BF16, gscale=None,
           round: int = FP4_ROUND_EVEN, mx_scale_rule: int = FP4_MX_SCALE_CEIL, out=None, workspace=None,
           weights_static: bool = False):
    """W4A4 linear from bf16 activations x (M x K) and a pre-quantized weight
    w = (Wq, Ws, gW) (N x K): quantizes x online, returns C = x W^T.
    ``weights_static``: w is written by no kernel still in flight (inference
    weights), so the decode kernel may stream it early."""
    import torch

    fmt = _fmt(fmt)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor, contiguous along K")
    _dev(x, "x", None, torch.bfloat16, contiguous=False)
    M, K = x.shape
    N = w[0].shape[0]
    Wq, Ws, gW = _operand(w, N, K, fmt, "W", x.device)
    if gscale is not None:
        _dev(gscale, "gscale", x.device, torch.float32, 4)
    dt = torch.float32 if out_dtype == FP4_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=x.device)
    _out2d(out, M, N, dt, "out", x.device)
    if workspace is None:
        workspace = torch.empty((linear_workspace_size(M, N, K, fmt),), dtype=torch.uint8, device=x.device)
    _dev(workspace, "workspace", x.device, torch.uint8)
    opts = _lib.Fp4Opts(int(round), int(mx_scale_rule), 0, 0, int(bool(weights_static)))
    _run("fp4_linear", x.device,
        x.data_ptr(), M, K, x.stride(0), fmt, int(hadamard_k), ctypes.byref(opts),
        gscale.data_ptr() if gscale is not None else None, Wq.data_ptr(), Ws.data_ptr(), gW.data_ptr(), N,
        int(out_dtype), out.data_ptr(), out.stride(0), workspace.data_ptr(), workspace.numel(),
        _stream_handle(torch, x.device))
    return out


def linear_residual(x, w, fmt, hadamard_k: int = 0, out_dtype: int = FP4_OUT_BF16, gscale=None,
                    round: int = FP4_ROUND_EVEN, mx_scale_rule: int = FP4_MX_SCALE_CEIL, out=None,
                    weights_static: bool = False):
    """The decode linear (M <= 16) with the sparse residual lane of TransFP4
    Eq.(3) in the activations (see fp4_linear_residual): each 32-value unit's
    largest rotated value (bf16) stays out of the FP4 stream and its product
    with W is added in the same launch.  w = (Wq, Ws, gW) as for
    :func:`linear`; no workspace."""
    import torch

    fmt = _fmt(fmt)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor, contiguous along K")
    _dev(x, "x", None, torch.bfloat16, contiguous=False)
    M, K = x.shape
    N = w[0].shape[0]
    Wq, Ws, gW = _operand(w, N, K, fmt, "W", x.device)
    if gscale is not None:
        _dev(gscale, "gscale", x.device, torch.float32, 4)
    dt = torch.float32 if out_dtype == FP4_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=x.device)
    _out2d(out, M, N, dt, "out", x.device)
    opts = _lib.Fp4Opts(int(round), int(mx_scale_rule), 0, 0, int(bool(weights_static)))
    _run("fp4_linear_residual", x.device,
         x.data_ptr(), M, K, x.stride(0), fmt, int(hadamard_k), ctypes.byref(opts),
         gscale.data_ptr() if gscale is not None else None, Wq.data_ptr(), Ws.data_ptr(), gW.data_ptr(), N,
         int(out_dtype), out.data_ptr(), out.stride(0), _stream_handle(torch, x.device))
    return out


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(_lib.lib().fp4_kernel_launches())


def check_device_status() -> None:
    import torch

    _lib.check("fp4_check_device_status",
               _lib.lib().fp4_check_device_status(_stream_handle(torch, torch.cuda.current_device())))
