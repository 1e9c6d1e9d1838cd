"""Python binding of librtq.so, the B200 weight-only quantized projection GEMM.

The functions named ``rt_*`` mirror the C ABI in include/rtq.h one to one and
only marshal arguments (raw pointers and sizes).  The helpers without the
prefix take torch tensors (device memory and streams are PyTorch's; every step
of the computation runs in the library's CUDA kernels) or numpy arrays (the
host quantizers) and raise :class:`RtqError` on any non-OK status.

There is no fallback: if librtq.so is missing or fails to load, every call
raises.  Build it with ``python -m int8_dequant_gemm_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

__all__ = [
    "RtqError", "lib", "PATHS", "OK", "qgemm_q4", "qgemm_q8", "qblock_project", "QBlock",
    "quantize_q4_g32", "quantize_q8_row", "dequant_q4_f32", "dequant_q8_f32",
    "dequant_q4_f16", "device_status", "auto_path", "status_string",
    "qgemm_noalloc", "plan", "block_fused", "workspace_bytes", "debug_inject",
    "qgemm_batch", "batch_plan", "Proj", "QBlockFmt", "qblock_project_fmt", "block_fused_fmt",
    "gemm_e4m3", "quantize_e4m3", "dequant_e4m3_f32", "dequant_e4m3_f16", "FMT_E4M3",
    "Checkpoint", "qgemm", "block_route", "ROUTE_GROUPED_SMALL_M", "ROUTE_X_RESIDENT_GROUP",
    "ROUTE_SIDE_PREPASS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librtq.so")

OK = 0
RT_ERR_INVALID_ARG = 1
RT_ERR_DEVICE_TIMEOUT = 5
RT_ERR_SCRATCH_LIMIT = 8
RT_ERR_OPERAND_RANGE = 9
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024   # RT_NOALLOC_SCRATCH_BYTES in include/rtq.h
PATHS = {"auto": 0, "simt": 1, "tc": 2}
FMT_E4M3, FMT_Q4, FMT_Q8 = 3, 4, 8     # rt_format

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_lib = None


class RtqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class _QProjC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("X", _p), ("Wq", _p),
                ("scales", _p), ("bias", _p), ("Y", _p), ("N", _i64), ("K", _i64)]


class _QWeightC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("Wq", _p), ("scales", _p),
                ("bias", _p)]


class _QBlockFmtC(ctypes.Structure):
    _fields_ = [("qkvg", _QWeightC), ("wo", _QWeightC), ("w13", _QWeightC), ("w2", _QWeightC),
                ("d_model", _i64), ("d_ff", _i64)]


class _StWeightC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("N", _i64), ("K", _i64),
                ("codes", _p), ("scales", _p), ("code_bytes", _i64), ("scale_bytes", _i64)]


class _QBlockC(ctypes.Structure):
    _fields_ = [("qkvg", _p), ("qkvg_sm", _p), ("wo", _p), ("wo_s", _p), ("w13", _p),
                ("w13_sm", _p), ("w2", _p), ("w2_s", _p), ("d_model", _i64), ("d_ff", _i64)]


def lib() -> ctypes.CDLL:
    """Loads librtq.so once; raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m int8_dequant_gemm_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.rt_status_string.restype = ctypes.c_char_p
    L.rt_status_string.argtypes = [_i32]
    L.rt_version.restype = _i32
    L.rt_version.argtypes = []
    for name in ("rt_qgemm_q4", "rt_qgemm_q8"):
        f = getattr(L, name)
        f.restype = _i32
        f.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _p]
    L.rt_qgemm.restype = _i32
    L.rt_qgemm.argtypes = [_i32, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i32, _p]
    L.rt_gemm_e4m3.restype = _i32
    L.rt_gemm_e4m3.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32, _p]
    L.rt_quantize_e4m3.restype = _i32
    L.rt_quantize_e4m3.argtypes = [_p, _i64, _p]
    for name in ("rt_dequant_e4m3_f32", "rt_dequant_e4m3_f16"):
        f = getattr(L, name)
        f.restype = _i32
        f.argtypes = [_p, _p, _i64, _i64, _p]
    L.rt_st_open.restype = _i32
    L.rt_st_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(_p)]
    L.rt_st_count.restype = _i64
    L.rt_st_count.argtypes = [_p]
    L.rt_st_weight_find.restype = _i32
    L.rt_st_weight_find.argtypes = [_p, ctypes.c_char_p, ctypes.POINTER(_StWeightC)]
    L.rt_st_close.restype = None
    L.rt_st_close.argtypes = [_p]
    L.rt_qgemm_noalloc.restype = _i32
    L.rt_qgemm_noalloc.argtypes = [_i32, _p, _p, _p, _p, _i64, _i64, _i64, _i32, _p]
    L.rt_qgemm_auto_path.restype = _i32
    L.rt_qgemm_auto_path.argtypes = [_i32, _i64, _i64, _i64]
    L.rt_qgemm_plan.restype = _i32
    L.rt_qgemm_plan.argtypes = [_i32, _i64, _i64, _i64, _i32]
    L.rt_workspace_bytes.restype = _i64
    L.rt_workspace_bytes.argtypes = [_i32, _i64, _i64, _i64, _i32]
    L.rt_workspace_reserve.restype = _i32
    L.rt_workspace_reserve.argtypes = [_i64, _p]
    L.rt_workspace_release.restype = _i32
    L.rt_workspace_release.argtypes = []
    L.rt_qblock_project.restype = _i32
    L.rt_qblock_project.argtypes = [ctypes.POINTER(_QBlockC), _i64, _p, _p, _p, _p, _p, _p, _p,
                                    _p, _i32, _p]
    L.rt_qblock_fused.restype = _i32
    L.rt_qblock_fused.argtypes = [_i64, _i64, _i64, _i32]
    L.rt_qblock_project_fmt.restype = _i32
    L.rt_qblock_project_fmt.argtypes = [ctypes.POINTER(_QBlockFmtC), _i64, _p, _p, _p, _p, _p, _p,
                                        _p, _p, _i32, _p]
    L.rt_qblock_fused_fmt.restype = _i32
    L.rt_qblock_fused_fmt.argtypes = [ctypes.POINTER(_QBlockFmtC), _i64, _i32]
    L.rt_qblock_route.restype = _i32
    L.rt_qblock_route.argtypes = [ctypes.POINTER(_QBlockC), _i64, _i32]
    L.rt_qblock_route_fmt.restype = _i32
    L.rt_qblock_route_fmt.argtypes = [ctypes.POINTER(_QBlockFmtC), _i64, _i32]
    L.rt_quantize_q4_g32.restype = _i32
    L.rt_quantize_q4_g32.argtypes = [_p, _i64, _i64, _i32, _p, _p]
    L.rt_quantize_q8_row.restype = _i32
    L.rt_quantize_q8_row.argtypes = [_p, _i64, _i64, _p, _p]
    for name in ("rt_dequant_q4_f32", "rt_dequant_q8_f32", "rt_dequant_q4_f16"):
        f = getattr(L, name)
        f.restype = _i32
        f.argtypes = [_p, _p, _p, _i64, _i64, _p]
    L.rt_device_status.restype = _i32
    L.rt_device_status.argtypes = [_p, ctypes.POINTER(_i32)]
    L.rt_debug_inject.restype = _i32
    L.rt_debug_inject.argtypes = [_i32, _i64]
    L.rt_qgemm_batch.restype = _i32
    L.rt_qgemm_batch.argtypes = [ctypes.POINTER(_QProjC), _i32, _i64, _i32, _p]
    L.rt_qgemm_batch_plan.restype = _i32
    L.rt_qgemm_batch_plan.argtypes = [ctypes.POINTER(_QProjC), _i32, _i64, _i32]
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().rt_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise RtqError(status, where)


# ----------------------------------------------------------------- raw ABI
def rt_qgemm_q4(X, Wq, scale_min, Y, M, N, K, path, stream) -> int:
    return lib().rt_qgemm_q4(X, Wq, scale_min, Y, M, N, K, path, stream)


def rt_qgemm_q8(X, Wq, scale, Y, M, N, K, path, stream) -> int:
    return lib().rt_qgemm_q8(X, Wq, scale, Y, M, N, K, path, stream)


def rt_qgemm(fmt, X, Wq, scales, bias, Y, M, N, K, path, stream) -> int:
    return lib().rt_qgemm(fmt, X, Wq, scales, bias, Y, M, N, K, path, stream)


def rt_gemm_e4m3(X, W, Y, M, N, K, path, stream) -> int:
    return lib().rt_gemm_e4m3(X, W, Y, M, N, K, path, stream)


def rt_quantize_e4m3(W, n, out) -> int:
    return lib().rt_quantize_e4m3(W, n, out)


def rt_dequant_e4m3_f32(Wq, W_out, N, K, stream) -> int:
    return lib().rt_dequant_e4m3_f32(Wq, W_out, N, K, stream)


def rt_dequant_e4m3_f16(Wq, W_out, N, K, stream) -> int:
    return lib().rt_dequant_e4m3_f16(Wq, W_out, N, K, stream)


def rt_qgemm_noalloc(fmt, X, Wq, scales, Y, M, N, K, path, stream) -> int:
    return lib().rt_qgemm_noalloc(fmt, X, Wq, scales, Y, M, N, K, path, stream)


def rt_qblock_project(blk, M, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13, Y_2, path,
                      stream) -> int:
    return lib().rt_qblock_project(ctypes.byref(blk), M, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o,
                                   Y_13, Y_2, path, stream)


def rt_qblock_fused(M, d_model, d_ff, path) -> int:
    return lib().rt_qblock_fused(M, d_model, d_ff, path)


def rt_qblock_project_fmt(blk, M, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13, Y_2, path,
                          stream) -> int:
    return lib().rt_qblock_project_fmt(ctypes.byref(blk), M, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg,
                                       Y_o, Y_13, Y_2, path, stream)


def rt_qblock_fused_fmt(blk, M, path) -> int:
    return lib().rt_qblock_fused_fmt(ctypes.byref(blk), M, path)


def rt_qblock_route(blk, M, path) -> int:
    return lib().rt_qblock_route(ctypes.byref(blk), M, path)


def rt_qblock_route_fmt(blk, M, path) -> int:
    return lib().rt_qblock_route_fmt(ctypes.byref(blk), M, path)


def rt_quantize_q4_g32(W, N, K, n_grid, Wq, scale_min) -> int:
    return lib().rt_quantize_q4_g32(W, N, K, n_grid, Wq, scale_min)


def rt_quantize_q8_row(W, N, K, Wq, scale) -> int:
    return lib().rt_quantize_q8_row(W, N, K, Wq, scale)


def rt_dequant_q4_f32(Wq, scale_min, W_out, N, K, stream) -> int:
    return lib().rt_dequant_q4_f32(Wq, scale_min, W_out, N, K, stream)


def rt_dequant_q8_f32(Wq, scale, W_out, N, K, stream) -> int:
    return lib().rt_dequant_q8_f32(Wq, scale, W_out, N, K, stream)


def rt_dequant_q4_f16(Wq, scale_min, W_out, N, K, stream) -> int:
    return lib().rt_dequant_q4_f16(Wq, scale_min, W_out, N, K, stream)


def rt_device_status(stream, out) -> int:
    return lib().rt_device_status(stream, out)


def rt_debug_inject(mode, wait_ns) -> int:
    return lib().rt_debug_inject(mode, wait_ns)


def rt_qgemm_batch(projs, count, M, path, stream) -> int:
    return lib().rt_qgemm_batch(projs, count, M, path, stream)


def rt_qgemm_batch_plan(projs, count, M, path) -> int:
    return lib().rt_qgemm_batch_plan(projs, count, M, path)


def rt_qgemm_auto_path(fmt, M, N, K) -> int:
    return lib().rt_qgemm_auto_path(fmt, M, N, K)


def rt_qgemm_plan(fmt, M, N, K, path) -> int:
    return lib().rt_qgemm_plan(fmt, M, N, K, path)


def rt_workspace_bytes(fmt, M, N, K, path) -> int:
    return lib().rt_workspace_bytes(fmt, M, N, K, path)


def rt_workspace_reserve(nbytes, stream) -> int:
    return lib().rt_workspace_reserve(nbytes, stream)


def rt_workspace_release() -> int:
    return lib().rt_workspace_release()


# ------------------------------------------------------- torch-level helpers
def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _path(path) -> int:
    return PATHS[path] if isinstance(path, str) else int(path)


def _shape(t, shape, name):
    """The C layer sees only pointers and sizes, so a tensor whose shape does
    not match the sizes would be read or written out of bounds: reject it."""
    got = tuple(t.shape)
    if got != tuple(shape):
        raise ValueError(f"{name} has shape {got}, expected {tuple(shape)}")


def _packed_shapes(fmt: int, N: int, K: int):
    """Shapes of the codes and the scales of an N x K weight in format q4 / q8
    (e4m3 has no scales: None)."""
    if fmt == 4:
        return (N, K // 2), (N, K // 32, 2)
    if fmt == FMT_E4M3:
        return (N, K), None
    return (N, K), (N,)


_DTYPES = {4: ("uint8", "uint16"), 8: ("int8", "float32"), FMT_E4M3: ("uint8", None)}


def _weight_ptrs(fmt, Wq, scales, name):
    """(codes, scales) pointers of one weight, dtypes checked (scales None for e4m3)."""
    import torch
    wdt, sdt = _DTYPES[fmt]
    w = _dev(Wq, getattr(torch, wdt), name)
    if sdt is None:
        return w, None
    return w, _dev(scales, getattr(torch, sdt), name + " scales")


def _check_gemm_shapes(fmt, X, Wq, scales, Y):
    if X.dim() != 2:
        raise ValueError(f"X must be 2-D [M, K], got shape {tuple(X.shape)}")
    M, K = X.shape
    N = Wq.shape[0]
    wshape, sshape = _packed_shapes(fmt, N, K)
    _shape(Wq, wshape, "Wq")
    if sshape is not None:
        _shape(scales, sshape, "scale_min" if fmt == 4 else "scale")
    if Y is not None:
        _shape(Y, (M, N), "Y")
    return M, N, K


def qgemm_q4(X, Wq, scale_min, Y=None, path="auto", stream=None):
    """Y[M,N] = X[M,K] @ dequant_q4(Wq[N,K/2], scale_min[N,K/32,2])^T on the GPU."""
    import torch
    M, N, K = _check_gemm_shapes(4, X, Wq, scale_min, Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    st = rt_qgemm_q4(_dev(X, torch.float32, "X"), _dev(Wq, torch.uint8, "Wq"),
                     _dev(scale_min, torch.uint16, "scale_min"), _dev(Y, torch.float32, "Y"),
                     M, N, K, _path(path), _stream_ptr(stream))
    _check(st, "rt_qgemm_q4")
    return Y


def qgemm_q8(X, Wq, scale, Y=None, path="auto", stream=None):
    """Y[M,N] = X[M,K] @ (Wq[N,K] * scale[N,None])^T on the GPU."""
    import torch
    M, N, K = _check_gemm_shapes(8, X, Wq, scale, Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    st = rt_qgemm_q8(_dev(X, torch.float32, "X"), _dev(Wq, torch.int8, "Wq"),
                     _dev(scale, torch.float32, "scale"), _dev(Y, torch.float32, "Y"),
                     M, N, K, _path(path), _stream_ptr(stream))
    _check(st, "rt_qgemm_q8")
    return Y


def qgemm(fmt, X, Wq, scales=None, bias=None, Y=None, path="auto", stream=None):
    """Y[M,N] = X[M,K] @ dequant(Wq, scales)^T + bias on the GPU, any format
    (4: q4, 8: q8, 3: e4m3 with scales None); bias: None or fp32 [N]."""
    import torch
    M, N, K = _check_gemm_shapes(fmt, X, Wq, scales, Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    b = None
    if bias is not None:
        _shape(bias, (N,), "bias")
        b = _dev(bias, torch.float32, "bias")
    w, sc = _weight_ptrs(fmt, Wq, scales, "Wq")
    st = rt_qgemm(fmt, _dev(X, torch.float32, "X"), w, sc, b, _dev(Y, torch.float32, "Y"),
                  M, N, K, _path(path), _stream_ptr(stream))
    _check(st, "rt_qgemm")
    return Y


def gemm_e4m3(X, W, Y=None, path="auto", stream=None):
    """Y[M,N] = X[M,K] @ e4m3(W[N,K])^T on the GPU (W: uint8 float8_e4m3fn codes)."""
    import torch
    M, N, K = _check_gemm_shapes(FMT_E4M3, X, W, None, Y)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    st = rt_gemm_e4m3(_dev(X, torch.float32, "X"), _dev(W, torch.uint8, "W"),
                      _dev(Y, torch.float32, "Y"), M, N, K, _path(path), _stream_ptr(stream))
    _check(st, "rt_gemm_e4m3")
    return Y


def qgemm_noalloc(fmt, X, Wq, scales, Y, path="auto", stream=None):
    """rt_qgemm_q4 (fmt 4) or rt_qgemm_q8 (fmt 8) into a caller-given Y, with the
    activation scratch in the library's fixed device array: no allocation."""
    import torch
    if fmt not in (4, 8):
        raise ValueError(f"fmt must be 4 or 8, got {fmt}")
    M, N, K = _check_gemm_shapes(fmt, X, Wq, scales, Y)
    wdt, sdt = (torch.uint8, torch.uint16) if fmt == 4 else (torch.int8, torch.float32)
    st = rt_qgemm_noalloc(fmt, _dev(X, torch.float32, "X"), _dev(Wq, wdt, "Wq"),
                          _dev(scales, sdt, "scales"), _dev(Y, torch.float32, "Y"),
                          M, N, K, _path(path), _stream_ptr(stream))
    _check(st, "rt_qgemm_noalloc")
    return Y


@dataclass
class Proj:
    """One entry of a projection list (see rt_qproj in rtq.h): fmt 4, 8 or 3,
    the device tensors X [M, K], Wq and scales in that format, Y [M, N], and
    an optional fp32 bias [N]."""
    fmt: int
    X: object
    Wq: object
    scales: object
    Y: object
    bias: object = None


def _batch_array(projs, M):
    import torch
    arr = (_QProjC * max(1, len(projs)))()
    for i, q in enumerate(projs):
        if q.fmt not in _DTYPES:
            raise ValueError(f"entry {i}: fmt must be 4, 8 or 3 (e4m3), got {q.fmt}")
        if q.X.dim() != 2 or q.X.shape[0] != M:
            raise ValueError(f"entry {i}: X must be [M={M}, K], got {tuple(q.X.shape)}")
        _, N, K = _check_gemm_shapes(q.fmt, q.X, q.Wq, q.scales, q.Y)
        w, sc = _weight_ptrs(q.fmt, q.Wq, q.scales, f"entry {i} Wq")
        b = None
        if q.bias is not None:
            _shape(q.bias, (N,), f"entry {i} bias")
            b = _dev(q.bias, torch.float32, "bias")
        arr[i] = _QProjC(q.fmt, 0, _dev(q.X, torch.float32, "X"), w, sc, b,
                         _dev(q.Y, torch.float32, "Y"), N, K)
    return arr


def qgemm_batch(projs, M=None, path="auto", stream=None):
    """Runs a list of independent projections with the same M (rt_qgemm_batch)."""
    if M is None:
        M = projs[0].X.shape[0] if projs else 0
    arr = _batch_array(projs, M)
    _check(rt_qgemm_batch(arr, len(projs), M, _path(path), _stream_ptr(stream)), "rt_qgemm_batch")


def batch_plan(projs, M=None, path="auto") -> str:
    """'tc_list' if rt_qgemm_batch runs the list as list launches, 'per_call'
    for one call per entry, 'rejected' otherwise."""
    if M is None:
        M = projs[0].X.shape[0] if projs else 0
    r = int(rt_qgemm_batch_plan(_batch_array(projs, M), len(projs), M, _path(path)))
    return {5: "tc_list", 0: "per_call"}.get(r, "rejected")


@dataclass
class QBlock:
    """Device tensors of one block's packed projections (see rt_qblock in rtq.h)."""
    qkvg: object
    qkvg_sm: object
    wo: object
    wo_s: object
    w13: object
    w13_sm: object
    w2: object
    w2_s: object
    d_model: int = 512
    d_ff: int = 2048

    def as_c(self) -> _QBlockC:
        import torch
        d, f = self.d_model, self.d_ff
        for (name, fmt, N, K) in (("qkvg", 4, 4 * d, d), ("wo", 8, d, d), ("w13", 4, 2 * f, d),
                                  ("w2", 8, d, f)):
            wshape, sshape = _packed_shapes(fmt, N, K)
            _shape(getattr(self, name), wshape, name)
            sname = name + ("_sm" if fmt == 4 else "_s")
            _shape(getattr(self, sname), sshape, sname)
        return _QBlockC(_dev(self.qkvg, torch.uint8, "qkvg"),
                        _dev(self.qkvg_sm, torch.uint16, "qkvg_sm"),
                        _dev(self.wo, torch.int8, "wo"), _dev(self.wo_s, torch.float32, "wo_s"),
                        _dev(self.w13, torch.uint8, "w13"),
                        _dev(self.w13_sm, torch.uint16, "w13_sm"),
                        _dev(self.w2, torch.int8, "w2"), _dev(self.w2_s, torch.float32, "w2_s"),
                        self.d_model, self.d_ff)


def qblock_project(block: QBlock, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13, Y_2,
                   path="auto", stream=None, block_c=None):
    """Runs one block's four quantized projections (qkvg, wo, w13, w2)."""
    import torch
    M = X_qkvg.shape[0]
    d, f = block.d_model, block.d_ff
    for t, shape, name in ((X_qkvg, (M, d), "X_qkvg"), (X_o, (M, d), "X_o"),
                           (X_ffn, (M, d), "X_ffn"), (X_w2, (M, f), "X_w2"),
                           (Y_qkvg, (M, 4 * d), "Y_qkvg"), (Y_o, (M, d), "Y_o"),
                           (Y_13, (M, 2 * f), "Y_13"), (Y_2, (M, d), "Y_2")):
        _shape(t, shape, name)
    bc = block_c if block_c is not None else block.as_c()
    args = [_dev(t, torch.float32, n) for t, n in
            ((X_qkvg, "X_qkvg"), (X_o, "X_o"), (X_ffn, "X_ffn"), (X_w2, "X_w2"),
             (Y_qkvg, "Y_qkvg"), (Y_o, "Y_o"), (Y_13, "Y_13"), (Y_2, "Y_2"))]
    st = rt_qblock_project(bc, M, *args, _path(path), _stream_ptr(stream))
    _check(st, "rt_qblock_project")


@dataclass
class QBlockFmt:
    """A block's four projections, each (fmt, Wq, scales) or (fmt, Wq, scales,
    bias) with fmt 4 (q4), 8 (q8) or 3 (e4m3, scales None), as device tensors
    (see rt_qblock_fmt in rtq.h).  All four q8 is the int8 card's all-int8
    recipe."""
    qkvg: tuple
    wo: tuple
    w13: tuple
    w2: tuple
    d_model: int = 512
    d_ff: int = 2048

    def as_c(self) -> _QBlockFmtC:
        import torch
        d, f = self.d_model, self.d_ff
        ws = []
        for name, N, K in (("qkvg", 4 * d, d), ("wo", d, d), ("w13", 2 * f, d), ("w2", d, f)):
            fmt, Wq, S, *rest = getattr(self, name)
            bias = rest[0] if rest else None
            if fmt not in _DTYPES:
                raise ValueError(f"{name}: fmt must be 4, 8 or 3 (e4m3), got {fmt}")
            wshape, sshape = _packed_shapes(fmt, N, K)
            _shape(Wq, wshape, name)
            if sshape is not None:
                _shape(S, sshape, name + " scales")
            b = None
            if bias is not None:
                _shape(bias, (N,), name + " bias")
                b = _dev(bias, torch.float32, name + " bias")
            ws.append(_QWeightC(fmt, 0, *_weight_ptrs(fmt, Wq, S, name), b))
        return _QBlockFmtC(*ws, d, f)


def _block_io(d, f, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13, Y_2):
    import torch
    M = X_qkvg.shape[0]
    for t, shape, name in ((X_qkvg, (M, d), "X_qkvg"), (X_o, (M, d), "X_o"),
                           (X_ffn, (M, d), "X_ffn"), (X_w2, (M, f), "X_w2"),
                           (Y_qkvg, (M, 4 * d), "Y_qkvg"), (Y_o, (M, d), "Y_o"),
                           (Y_13, (M, 2 * f), "Y_13"), (Y_2, (M, d), "Y_2")):
        _shape(t, shape, name)
    return M, [_dev(t, torch.float32, n) for t, n in
               ((X_qkvg, "X_qkvg"), (X_o, "X_o"), (X_ffn, "X_ffn"), (X_w2, "X_w2"),
                (Y_qkvg, "Y_qkvg"), (Y_o, "Y_o"), (Y_13, "Y_13"), (Y_2, "Y_2"))]


def qblock_project_fmt(block: QBlockFmt, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13, Y_2,
                       path="auto", stream=None):
    """Runs one block's four projections with per-projection formats."""
    M, args = _block_io(block.d_model, block.d_ff, X_qkvg, X_o, X_ffn, X_w2, Y_qkvg, Y_o, Y_13,
                        Y_2)
    st = rt_qblock_project_fmt(block.as_c(), M, *args, _path(path), _stream_ptr(stream))
    _check(st, "rt_qblock_project_fmt")


def block_fused_fmt(block: QBlockFmt, M: int, path="auto") -> int:
    return int(rt_qblock_fused_fmt(block.as_c(), M, _path(path)))


# rt_route bits (see rt_qblock_route in rtq.h)
ROUTE_GROUPED_SMALL_M, ROUTE_X_RESIDENT_GROUP, ROUTE_SIDE_PREPASS = 1, 2, 4


def block_route(block, M: int, path="auto") -> int:
    """How the block driver runs `block` (a QBlock or QBlockFmt) at M rows: a
    sum of the ROUTE_* bits, 0 for one call per projection, -1 if rejected."""
    if isinstance(block, QBlockFmt):
        return int(rt_qblock_route_fmt(block.as_c(), M, _path(path)))
    return int(rt_qblock_route(block.as_c(), M, _path(path)))


def quantize_q4_g32(W: np.ndarray, n_grid: int = 21):
    """Host min-MSE g32 quantizer: (Wq uint8 [N,K/2], scale_min uint16 [N,K/32,2])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.empty((N, K // 2), dtype=np.uint8)
    sm = np.empty((N, K // 32, 2), dtype=np.uint16)
    st = rt_quantize_q4_g32(W.ctypes.data, N, K, n_grid, Wq.ctypes.data, sm.ctypes.data)
    _check(st, "rt_quantize_q4_g32")
    return Wq, sm


def quantize_e4m3(W: np.ndarray) -> np.ndarray:
    """Host FP8 quantizer: float8_e4m3fn codes (uint8, same shape as W)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out = np.empty(W.shape, dtype=np.uint8)
    _check(rt_quantize_e4m3(W.ctypes.data, W.size, out.ctypes.data), "rt_quantize_e4m3")
    return out


def dequant_e4m3_f32(Wq, stream=None):
    import torch
    N, K = Wq.shape
    out = torch.empty((N, K), dtype=torch.float32, device=Wq.device)
    _check(rt_dequant_e4m3_f32(_dev(Wq, torch.uint8, "Wq"), _dev(out, torch.float32, "W_out"),
                               N, K, _stream_ptr(stream)), "rt_dequant_e4m3_f32")
    return out


def dequant_e4m3_f16(Wq, stream=None):
    """The tensor-core operand of e4m3 weights, as fp16 bits (uint16) [N, K]."""
    import torch
    N, K = Wq.shape
    out = torch.empty((N, K), dtype=torch.uint16, device=Wq.device)
    _check(rt_dequant_e4m3_f16(_dev(Wq, torch.uint8, "Wq"), _dev(out, torch.uint16, "W_out"),
                               N, K, _stream_ptr(stream)), "rt_dequant_e4m3_f16")
    return out


def quantize_q8_row(W: np.ndarray):
    """Host per-row int8 quantizer: (Wq int8 [N,K], scale float32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), dtype=np.int8)
    sc = np.empty((N,), dtype=np.float32)
    st = rt_quantize_q8_row(W.ctypes.data, N, K, Wq.ctypes.data, sc.ctypes.data)
    _check(st, "rt_quantize_q8_row")
    return Wq, sc


def dequant_q4_f32(Wq, scale_min, stream=None):
    import torch
    N, K2 = Wq.shape
    _shape(scale_min, _packed_shapes(4, N, 2 * K2)[1], "scale_min")
    out = torch.empty((N, 2 * K2), dtype=torch.float32, device=Wq.device)
    st = rt_dequant_q4_f32(_dev(Wq, torch.uint8, "Wq"), _dev(scale_min, torch.uint16, "scale_min"),
                           _dev(out, torch.float32, "W_out"), N, 2 * K2, _stream_ptr(stream))
    _check(st, "rt_dequant_q4_f32")
    return out


def dequant_q4_f16(Wq, scale_min, stream=None):
    """fp16 rendering of the q4 weights (the tensor-core operand) as uint16 bits [N, K]."""
    import torch
    N, K2 = Wq.shape
    _shape(scale_min, _packed_shapes(4, N, 2 * K2)[1], "scale_min")
    out = torch.empty((N, 2 * K2), dtype=torch.uint16, device=Wq.device)
    st = rt_dequant_q4_f16(_dev(Wq, torch.uint8, "Wq"), _dev(scale_min, torch.uint16, "scale_min"),
                           _dev(out, torch.uint16, "W_out"), N, 2 * K2, _stream_ptr(stream))
    _check(st, "rt_dequant_q4_f16")
    return out


def dequant_q8_f32(Wq, scale, stream=None):
    import torch
    N, K = Wq.shape
    _shape(scale, (N,), "scale")
    out = torch.empty((N, K), dtype=torch.float32, device=Wq.device)
    st = rt_dequant_q8_f32(_dev(Wq, torch.int8, "Wq"), _dev(scale, torch.float32, "scale"),
                           _dev(out, torch.float32, "W_out"), N, K, _stream_ptr(stream))
    _check(st, "rt_dequant_q8_f32")
    return out


def device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device status word:
    OK, RT_ERR_DEVICE_TIMEOUT or RT_ERR_OPERAND_RANGE."""
    v = ctypes.c_int(0)
    _check(rt_device_status(_stream_ptr(stream), ctypes.byref(v)), "rt_device_status")
    return int(v.value)


def debug_inject(mode: int, wait_ns: int = 0):
    """Test hook of the device failure path (see rt_debug_inject): mode 1 makes
    the first producer arrival of every CTA go missing, with every bounded wait
    limited to wait_ns; debug_inject(0) restores normal operation."""
    _check(rt_debug_inject(int(mode), int(wait_ns)), "rt_debug_inject")


def auto_path(fmt: int, M: int, N: int, K: int) -> int:
    return int(rt_qgemm_auto_path(fmt, M, N, K))


KERNELS = {1: "simt", 2: "tc_w_stationary", 3: "tc_x_resident", 4: "tc_w_streamed", 5: "tc_list",
           6: "tc_x_resident_pair"}


def plan(fmt: int, M: int, N: int, K: int, path="auto") -> str:
    """Name of the kernel a GEMM of this shape runs (see rt_qgemm_plan)."""
    k = int(rt_qgemm_plan(fmt, M, N, K, _path(path)))
    return KERNELS.get(k, "rejected")


def block_fused(M: int, d_model: int, d_ff: int, path="auto") -> int:
    """1 if rt_qblock_project runs the block as one grouped launch, 0 if one
    call per projection, -1 if it rejects the sizes (see rt_qblock_fused)."""
    return int(rt_qblock_fused(M, d_model, d_ff, _path(path)))


def workspace_bytes(fmt: int, M: int, N: int, K: int, path="auto") -> int:
    return int(rt_workspace_bytes(fmt, M, N, K, _path(path)))


def workspace_reserve(nbytes: int, stream=None):
    _check(rt_workspace_reserve(int(nbytes), _stream_ptr(stream)), "rt_workspace_reserve")


def workspace_release():
    _check(rt_workspace_release(), "rt_workspace_release")


class Checkpoint:
    """A quantized checkpoint file (plain safetensors) read through rt_st_*:
    ``weight(name)`` returns (fmt, codes, scales) as host numpy arrays in the
    layouts the GEMMs take (q4: uint8 [N, K/2] + uint16 [N, K/32, 2]; q8:
    int8 [N, K] + float32 [N]; e4m3: uint8 [N, K] + None), the format detected
    from the dtypes."""

    def __init__(self, path):
        self._h = ctypes.c_void_p()
        _check(lib().rt_st_open(os.fsencode(path), ctypes.byref(self._h)), "rt_st_open")

    def __len__(self):
        return int(lib().rt_st_count(self._h))

    def weight(self, name: str):
        w = _StWeightC()
        _check(lib().rt_st_weight_find(self._h, name.encode(), ctypes.byref(w)),
               f"rt_st_weight_find({name})")
        N, K, fmt = int(w.N), int(w.K), int(w.fmt)
        codes = np.frombuffer(ctypes.string_at(w.codes, w.code_bytes), dtype=np.uint8)
        if fmt == FMT_Q4:
            sc = np.frombuffer(ctypes.string_at(w.scales, w.scale_bytes), dtype=np.uint16)
            return fmt, codes.reshape(N, K // 2).copy(), sc.reshape(N, K // 32, 2).copy()
        if fmt == FMT_Q8:
            sc = np.frombuffer(ctypes.string_at(w.scales, w.scale_bytes), dtype=np.float32)
            return fmt, codes.view(np.int8).reshape(N, K).copy(), sc.copy()
        return fmt, codes.reshape(N, K).copy(), None

    def close(self):
        if self._h:
            lib().rt_st_close(self._h)
            self._h = ctypes.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
