"""ctypes binding of libfp4.so (C ABI in include/fp4.h).

Argument marshalling only: every step of quantization and GEMM runs in the
library's CUDA kernels.  Pointer arguments take a torch tensor (its
``data_ptr()``), an integer address or None; ``stream`` defaults to torch's
current CUDA stream.  A non-OK status raises :class:`Fp4Error`.

Importing this module loads the library and raises ImportError if it has not
been built (``python -m fp4_block_scaled_h16_b200.build``): there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libfp4.so is not built: run `python -m fp4_block_scaled_h16_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

# enums (include/fp4.h)
FP4_OK, FP4_ERR_INVALID_ARG, FP4_ERR_UNSUPPORTED_SHAPE, FP4_ERR_MISALIGNED = 0, 1, 2, 3
FP4_ERR_WORKSPACE, FP4_ERR_NO_DEVICE, FP4_ERR_CUDA, FP4_ERR_TIMEOUT, FP4_ERR_UNSUPPORTED = 4, 5, 6, 7, 8
FP4_MXFP4, FP4_NVFP4, FP4_UFP4 = 0, 1, 2
FP4_RTNE, FP4_SR = 0, 1
FP4_ROT_NONE, FP4_ROT_H16, FP4_ROT_H32, FP4_ROT_RH16, FP4_ROT_RH32 = 0, 1, 2, 3, 4
FP4_IN_F32, FP4_IN_BF16 = 0, 1
FP4_OUT_F32, FP4_OUT_BF16 = 0, 1

EXPORTS = ("fp4_scales_bytes", "fp4_quantize_workspace_size", "fp4_amax", "fp4_quantize",
           "fp4_gemm", "fp4_last_error", "fp4_status_string", "fp4_set_wait_limit",
           "fp4_quantize_noalloc", "fp4_requantize", "fp4_rotate", "fp4_mxnorm_quantize",
           "fp4_gemm_workspace_size", "fp4_channel_amax", "fp4_outctl_workspace_size", "fp4_outctl_quantize",
           "fp4_gemm_outctl", "fp4_set_gemm_cta_pairs", "fp4_quantize_both_axes")

_P, _I, _I64, _U64, _U32, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                 ctypes.c_uint32, ctypes.c_size_t)
_lib.fp4_status_string.argtypes = [_I]
_lib.fp4_status_string.restype = ctypes.c_char_p
_lib.fp4_scales_bytes.argtypes = [_I64, _I64, _I]
_lib.fp4_scales_bytes.restype = _SZ
_lib.fp4_quantize_workspace_size.argtypes = [_I, _I, _I, ctypes.POINTER(_SZ)]
_lib.fp4_amax.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _U64, _P, _P]
_lib.fp4_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _I, _I, _I, _U64, _U32, _P,
                              _P, _P, _P, _P, _P, _SZ, _P]
_lib.fp4_quantize_both_axes.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _U64, _I, _U32, _P, _P, _P, _I, _U32, _P,
                                        _P, _P, _P, _SZ, _P]
_lib.fp4_quantize_noalloc.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _I, _I, _U64, _U32, _P, _P, _P, _P]
_lib.fp4_requantize.argtypes = [_P, _P, _P, _P, _I64, _I64, _I, _I, _I, _I, _I, _I, _U64, _U32, _P, _P, _P, _P, _P,
                                _P, _SZ, _P]
_lib.fp4_mxnorm_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _I, ctypes.c_float, _U64, _U32, _P, _P, _P,
                                     _P, _P, _SZ, _P]
_lib.fp4_channel_amax.argtypes = [_P, _I, _I64, _I64, _I64, _P, _P]
_lib.fp4_outctl_workspace_size.argtypes = [_I64, ctypes.POINTER(_SZ)]
_lib.fp4_outctl_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I64, _I64, _I, _I, _U64, _U32, _P, _P, _P, _P, _P,
                                     _P, _SZ, _P]
_lib.fp4_gemm_outctl.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _I, _I64, _P]
_lib.fp4_rotate.argtypes = [_P, _I, _I64, _I64, _I64, _I, _I, _U64, _P, _I64, _P]
_lib.fp4_gemm.argtypes = [_I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I, _I64, _P, _SZ, _P]
_lib.fp4_gemm_workspace_size.argtypes = [_I, _I, _I64, _I64, _I64, ctypes.POINTER(_SZ)]
_lib.fp4_last_error.argtypes = [_P]
_lib.fp4_set_wait_limit.argtypes = [_U32]
_lib.fp4_set_wait_limit.restype = None
_lib.fp4_set_gemm_cta_pairs.argtypes = [_I]
_lib.fp4_set_gemm_cta_pairs.restype = None
for _f in ("fp4_amax", "fp4_rotate", "fp4_mxnorm_quantize", "fp4_gemm_workspace_size", "fp4_channel_amax",
           "fp4_outctl_workspace_size", "fp4_outctl_quantize", "fp4_gemm_outctl", "fp4_quantize", "fp4_quantize_noalloc",
           "fp4_quantize_both_axes", "fp4_requantize", "fp4_gemm", "fp4_last_error",
           "fp4_quantize_workspace_size"):
    getattr(_lib, _f).restype = _I


class Fp4Error(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__("%s%s" % (where + ": " if where else "", fp4_status_string(status)))


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != FP4_OK:
        raise Fp4Error(status, where)


def fp4_status_string(status: int) -> str:
    return _lib.fp4_status_string(status).decode()


def fp4_scales_bytes(lines: int, K: int, fmt: int) -> int:
    return _lib.fp4_scales_bytes(lines, K, fmt)


def fp4_quantize_workspace_size(fmt: int, double_block: bool, amax_given: bool) -> int:
    n = _SZ(0)
    _check(_lib.fp4_quantize_workspace_size(fmt, int(double_block), int(amax_given), ctypes.byref(n)),
           "fp4_quantize_workspace_size")
    return n.value


def fp4_set_wait_limit(polls: int) -> None:
    _lib.fp4_set_wait_limit(polls)


def fp4_set_gemm_cta_pairs(enable: bool) -> None:
    _lib.fp4_set_gemm_cta_pairs(int(bool(enable)))


def fp4_amax(x, in_dtype, rows, cols, ld, rotation, axis, seed, amax_out, stream=None) -> None:
    _check(_lib.fp4_amax(_ptr(x), in_dtype, rows, cols, ld, rotation, axis, seed, _ptr(amax_out),
                         _stream(stream)), "fp4_amax")


def fp4_rotate(x, in_dtype, rows, cols, ld, rotation, axis, seed, y, ldy, stream=None) -> None:
    _check(_lib.fp4_rotate(_ptr(x), in_dtype, rows, cols, ld, rotation, axis, seed, _ptr(y), ldy,
                           _stream(stream)), "fp4_rotate")


def rotate(x, rotation, seed=0, out=None, stream=None):
    """The rotation alone along the rows of a 2-D CUDA tensor, in its own dtype (fp4_rotate)."""
    import torch
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    y = out if out is not None else torch.empty((rows, cols), dtype=x.dtype, device=x.device)
    fp4_rotate(x, in_dtype_of(x), rows, cols, ld, rotation, 1, seed, y, y.stride(0) if rows > 1 else cols, stream)
    return y


def fp4_mxnorm_quantize(x, in_dtype, rows, cols, ld, fmt, rounding, p, c, seed, tensor_id, codes, scales,
                        tensor_scale, rho, workspace, workspace_bytes, stream=None) -> None:
    _check(_lib.fp4_mxnorm_quantize(_ptr(x), in_dtype, rows, cols, ld, fmt, rounding, p, c, seed, tensor_id,
                                    _ptr(codes), _ptr(scales), _ptr(tensor_scale), _ptr(rho), _ptr(workspace),
                                    workspace_bytes, _stream(stream)), "fp4_mxnorm_quantize")


def mxnorm_quantize(x, fmt, p, c, rounding=FP4_RTNE, seed=0, tensor_id=0, out=None, rho=None, workspace=None,
                    stream=None):
    """MXNorm fused with the cast of a 2-D CUDA tensor along its rows
    (fp4_mxnorm_quantize): returns the quantized tensor with its "rho" [rows]."""
    import torch
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    q = out if out is not None else alloc_qtensor(rows, cols, fmt, False, x.device)
    r = rho if rho is not None else torch.empty(max(rows, 1), dtype=torch.float32, device=x.device)
    ws_bytes = 0 if fmt == FP4_MXFP4 else 256
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    fp4_mxnorm_quantize(x, in_dtype_of(x), rows, cols, ld, fmt, rounding, p, c, seed, tensor_id, q["codes"],
                        q["scales"], q["tensor_scale"], r, workspace if ws_bytes else None, ws_bytes, stream)
    q["rho"] = r
    return q


def fp4_quantize(x, in_dtype, rows, cols, ld, fmt, rounding, rotation, axis, double_block, seed,
                 tensor_id, tensor_amax, codes, scales, outer_scales, tensor_scale, workspace,
                 workspace_bytes, stream=None) -> None:
    _check(_lib.fp4_quantize(_ptr(x), in_dtype, rows, cols, ld, fmt, rounding, rotation, axis,
                             int(double_block), seed, tensor_id, _ptr(tensor_amax), _ptr(codes),
                             _ptr(scales), _ptr(outer_scales), _ptr(tensor_scale), _ptr(workspace),
                             workspace_bytes, _stream(stream)), "fp4_quantize")


def fp4_requantize(src_codes, src_scales, src_outer, src_tensor_scale, lines, K, src_fmt, src_double_block,
                   fmt, rounding, rotation, double_block, seed, tensor_id, tensor_amax, codes, scales,
                   outer_scales, tensor_scale, workspace, workspace_bytes, stream=None) -> None:
    _check(_lib.fp4_requantize(_ptr(src_codes), _ptr(src_scales), _ptr(src_outer), _ptr(src_tensor_scale),
                               lines, K, src_fmt, int(src_double_block), fmt, rounding, rotation,
                               int(double_block), seed, tensor_id, _ptr(tensor_amax), _ptr(codes), _ptr(scales),
                               _ptr(outer_scales), _ptr(tensor_scale), _ptr(workspace), workspace_bytes,
                               _stream(stream)), "fp4_requantize")


def requantize(q, fmt, rounding=FP4_RTNE, rotation=FP4_ROT_NONE, double_block=False, seed=0, tensor_id=0,
               tensor_amax=None, out=None, workspace=None, stream=None):
    """Re-quantize the quantized tensor q (lines x K) along the other axis: the
    result has K lines of q["lines"] elements (fp4_requantize)."""
    import torch
    lines, K = q["lines"], q["K"]
    r = out if out is not None else alloc_qtensor(K, lines, fmt, double_block, q["codes"].device)
    ws_bytes = fp4_quantize_workspace_size(fmt, double_block, tensor_amax is not None)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q["codes"].device)
    fp4_requantize(q["codes"], q["scales"], q["outer"], q["tensor_scale"] if q["format"] != FP4_MXFP4 else None,
                   lines, K, q["format"], q["double_block"], fmt, rounding, rotation, double_block, seed,
                   tensor_id, tensor_amax, r["codes"], r["scales"], r["outer"], r["tensor_scale"],
                   workspace if ws_bytes else None, ws_bytes, stream)
    return r


def fp4_quantize_noalloc(x, in_dtype, rows, cols, ld, fmt, rounding, rotation, axis, seed, tensor_id,
                         codes, scales, tensor_scale, stream=None) -> None:
    """fp4_quantize (NVFP4 / UFP4, internal amax) without a workspace: the
    scratch is the library's static device array.  For callers that cannot
    allocate device memory; concurrent calls race on that array."""
    _check(_lib.fp4_quantize_noalloc(_ptr(x), in_dtype, rows, cols, ld, fmt, rounding, rotation, axis, seed,
                                     tensor_id, _ptr(codes), _ptr(scales), _ptr(tensor_scale), _stream(stream)),
           "fp4_quantize_noalloc")


def fp4_gemm_workspace_size(fmt: int, double_block: bool, M: int, N: int, K: int) -> int:
    n = _SZ(0)
    _check(_lib.fp4_gemm_workspace_size(fmt, int(double_block), M, N, K, ctypes.byref(n)), "fp4_gemm_workspace_size")
    return n.value


def fp4_gemm(fmt, double_block, a_codes, a_scales, a_outer, a_tensor_scale, b_codes, b_scales,
             b_outer, b_tensor_scale, M, N, K, c, out_dtype, ldc, workspace=None, workspace_bytes=0,
             stream=None) -> None:
    _check(_lib.fp4_gemm(fmt, int(double_block), _ptr(a_codes), _ptr(a_scales), _ptr(a_outer),
                         _ptr(a_tensor_scale), _ptr(b_codes), _ptr(b_scales), _ptr(b_outer),
                         _ptr(b_tensor_scale), M, N, K, _ptr(c), out_dtype, ldc, _ptr(workspace),
                         workspace_bytes, _stream(stream)),
           "fp4_gemm")


def fp4_last_error(stream=None) -> int:
    """Status of the device error word (FP4_OK or FP4_ERR_TIMEOUT); clears it."""
    return _lib.fp4_last_error(_stream(stream))


# --------------------------------------------------------------------------- helpers
# Device buffers for a quantized tensor, allocated with torch (plumbing only).

def in_dtype_of(x) -> int:
    import torch
    if x.dtype == torch.bfloat16:
        return FP4_IN_BF16
    if x.dtype == torch.float32:
        return FP4_IN_F32
    raise TypeError("input must be bfloat16 or float32, got %s" % x.dtype)


def alloc_qtensor(lines: int, K: int, fmt: int, double_block: bool = False, device="cuda"):
    """codes [L, K/2] u8, tiled scales, outer [L, K/128] f32 (double block), tensor scale f32."""
    import torch
    return dict(
        codes=torch.empty((lines, K // 2), dtype=torch.uint8, device=device),
        scales=torch.empty(max(fp4_scales_bytes(lines, K, fmt), 16), dtype=torch.uint8, device=device),
        outer=torch.empty((lines, max(K // 128, 1)), dtype=torch.float32, device=device) if double_block else None,
        tensor_scale=torch.empty(1, dtype=torch.float32, device=device),
        lines=lines, K=K, format=fmt, double_block=bool(double_block))


def quantize(x, fmt, rounding=FP4_RTNE, rotation=FP4_ROT_NONE, axis=1, double_block=False, seed=0,
             tensor_id=0, tensor_amax=None, out=None, workspace=None, cols=None, stream=None):
    """Quantize a 2-D CUDA tensor (row-major, unit stride in the last dim) into a new or given qtensor."""
    import torch
    rows, ld = x.shape[0], x.stride(0) if x.dim() == 2 and x.shape[0] > 1 else x.shape[1]
    cols = x.shape[1] if cols is None else cols
    K, L = (cols, rows) if axis == 1 else (rows, cols)
    q = out if out is not None else alloc_qtensor(L, K, fmt, double_block, x.device)
    ws_bytes = fp4_quantize_workspace_size(fmt, double_block, tensor_amax is not None)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    fp4_quantize(x, in_dtype_of(x), rows, cols, ld, fmt, rounding, rotation, axis, double_block, seed,
                 tensor_id, tensor_amax, q["codes"], q["scales"], q["outer"], q["tensor_scale"],
                 workspace if ws_bytes else None, ws_bytes, stream)
    return q


def fp4_quantize_both_axes(x, in_dtype, rows, cols, ld, fmt, rotation, seed, rounding_rows, tensor_id_rows,
                           codes_rows, scales_rows, tensor_scale_rows, rounding_cols, tensor_id_cols, codes_cols,
                           scales_cols, tensor_scale_cols, workspace, workspace_bytes, stream=None) -> None:
    _check(_lib.fp4_quantize_both_axes(_ptr(x), in_dtype, rows, cols, ld, fmt, rotation, seed, rounding_rows,
                                       tensor_id_rows, _ptr(codes_rows), _ptr(scales_rows), _ptr(tensor_scale_rows),
                                       rounding_cols, tensor_id_cols, _ptr(codes_cols), _ptr(scales_cols),
                                       _ptr(tensor_scale_cols), _ptr(workspace), workspace_bytes, _stream(stream)),
           "fp4_quantize_both_axes")


def quantize_both_axes(x, fmt, rotation=FP4_ROT_NONE, seed=0, rounding_rows=FP4_RTNE, tensor_id_rows=0,
                       rounding_cols=FP4_RTNE, tensor_id_cols=0, out_rows=None, out_cols=None, workspace=None,
                       stream=None):
    """Quantize a 2-D bf16 CUDA tensor along its rows and its columns in one pass;
    returns (qtensor of the rows, qtensor of the columns)."""
    import torch
    rows, cols = x.shape
    ld = x.stride(0) if rows > 1 else cols
    qr = out_rows if out_rows is not None else alloc_qtensor(rows, cols, fmt, False, x.device)
    qc = out_cols if out_cols is not None else alloc_qtensor(cols, rows, fmt, False, x.device)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=x.device)
    fp4_quantize_both_axes(x, in_dtype_of(x), rows, cols, ld, fmt, rotation, seed, rounding_rows, tensor_id_rows,
                           qr["codes"], qr["scales"], qr["tensor_scale"], rounding_cols, tensor_id_cols,
                           qc["codes"], qc["scales"], qc["tensor_scale"], workspace, workspace.numel(), stream)
    return qr, qc


def gemm(qa, qb, out_dtype=FP4_OUT_F32, out=None, workspace=None, stream=None):
    """C = A B^T on two quantized tensors of the same format (lines along K);
    UFP4 takes a workspace (allocated here when none is given)."""
    import torch
    M, N, K = qa["lines"], qb["lines"], qa["K"]
    if qb["K"] != K or qa["format"] != qb["format"] or qa["double_block"] != qb["double_block"]:
        raise ValueError("operands must share K, format and double-block mode")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16 if out_dtype == FP4_OUT_BF16 else torch.float32,
                          device=qa["codes"].device)
    ws_bytes = fp4_gemm_workspace_size(qa["format"], qa["double_block"], M, N, K)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=qa["codes"].device)
    fp4_gemm(qa["format"], qa["double_block"], qa["codes"], qa["scales"], qa["outer"], qa["tensor_scale"],
             qb["codes"], qb["scales"], qb["outer"], qb["tensor_scale"], M, N, K, out, out_dtype,
             out.stride(0), workspace if ws_bytes else None, ws_bytes, stream)
    return out


# --------------------------------------------------------------------------- OutControl

def fp4_channel_amax(x, in_dtype, rows, cols, ld, amax_out, stream=None) -> None:
    _check(_lib.fp4_channel_amax(_ptr(x), in_dtype, rows, cols, ld, _ptr(amax_out), _stream(stream)),
           "fp4_channel_amax")


def fp4_outctl_workspace_size(cols: int) -> int:
    n = _SZ(0)
    _check(_lib.fp4_outctl_workspace_size(cols, ctypes.byref(n)), "fp4_outctl_workspace_size")
    return n.value


def fp4_outctl_quantize(x, in_dtype, rows, cols, ld, channels, n_channels, k8, rounding, rotation, seed, tensor_id,
                        codes, scales, tensor_scale, codes8, scale8, workspace, workspace_bytes, stream=None) -> None:
    _check(_lib.fp4_outctl_quantize(_ptr(x), in_dtype, rows, cols, ld, _ptr(channels), n_channels, k8, rounding,
                                    rotation, seed, tensor_id, _ptr(codes), _ptr(scales), _ptr(tensor_scale),
                                    _ptr(codes8), _ptr(scale8), _ptr(workspace), workspace_bytes, _stream(stream)),
           "fp4_outctl_quantize")


def fp4_gemm_outctl(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, a8_codes, a8_scale, b8_codes, b8_scale,
                    M, N, K, K8, c, out_dtype, ldc, stream=None) -> None:
    _check(_lib.fp4_gemm_outctl(_ptr(a_codes), _ptr(a_scales), _ptr(a_ts), _ptr(b_codes), _ptr(b_scales), _ptr(b_ts),
                                _ptr(a8_codes), _ptr(a8_scale), _ptr(b8_codes), _ptr(b8_scale), M, N, K, K8, _ptr(c),
                                out_dtype, ldc, _stream(stream)), "fp4_gemm_outctl")


def channel_amax(x, stream=None):
    """max over rows of |x[:, c]| for a 2-D CUDA tensor (fp4_channel_amax)."""
    import torch
    rows, cols = x.shape
    out = torch.empty(max(cols, 1), dtype=torch.float32, device=x.device)
    fp4_channel_amax(x, in_dtype_of(x), rows, cols, x.stride(0) if rows > 1 else cols, out, stream)
    return out[:cols]


def outctl_channels(amax, p: float):
    """Calibration: the ceil(p * cols) channels with the largest amax (ties to
    the lower index), in ascending order, as a device int32 tensor."""
    import math
    import torch
    n = math.ceil(p * amax.numel())
    order = torch.sort(-amax, stable=True).indices[:n]
    return torch.sort(order).values.to(torch.int32)


def outctl_quantize(x, channels, k8=None, rounding=FP4_RTNE, rotation=FP4_ROT_NONE, seed=0, tensor_id=0,
                    out=None, stream=None):
    """The OutControl split of a 2-D CUDA tensor along its channels
    (fp4_outctl_quantize): {"fp4": NVFP4 qtensor, "fp8": {"codes", "scale", "K"}}."""
    import torch
    rows, cols = x.shape
    n = channels.numel()
    k8 = (n + 127) // 128 * 128 if k8 is None else k8
    o = out if out is not None else dict(
        fp4=alloc_qtensor(rows, cols, FP4_NVFP4, False, x.device),
        fp8=dict(codes=torch.empty((rows, max(k8, 1)), dtype=torch.uint8, device=x.device),
                 scale=torch.empty(1, dtype=torch.float32, device=x.device), K=k8))
    ws = torch.empty(fp4_outctl_workspace_size(cols), dtype=torch.uint8, device=x.device)
    q4, q8 = o["fp4"], o["fp8"]
    fp4_outctl_quantize(x, in_dtype_of(x), rows, cols, x.stride(0) if rows > 1 else cols, channels, n, k8, rounding,
                        rotation, seed, tensor_id, q4["codes"], q4["scales"], q4["tensor_scale"], q8["codes"],
                        q8["scale"], ws, ws.numel(), stream)
    return o


def gemm_outctl(qa, qb, out_dtype=FP4_OUT_F32, out=None, stream=None):
    """C = A B^T on two OutControl-split operands (fp4_gemm_outctl)."""
    import torch
    a4, b4, a8, b8 = qa["fp4"], qb["fp4"], qa["fp8"], qb["fp8"]
    M, N, K, K8 = a4["lines"], b4["lines"], a4["K"], a8["K"]
    if b4["K"] != K or b8["K"] != K8:
        raise ValueError("operands must share K and the FP8 width")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16 if out_dtype == FP4_OUT_BF16 else torch.float32,
                          device=a4["codes"].device)
    fp4_gemm_outctl(a4["codes"], a4["scales"], a4["tensor_scale"], b4["codes"], b4["scales"], b4["tensor_scale"],
                    a8["codes"], a8["scale"], b8["codes"], b8["scale"], M, N, K, K8, out, out_dtype, out.stride(0),
                    stream)
    return out
