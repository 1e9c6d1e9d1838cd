"""Double-precision CPU oracle for the weight-only quantized projection GEMM.

TEST INFRASTRUCTURE ONLY: the test-suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this module, and this module imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, IEEE double); this file only
builds it with gcc and marshals numpy arrays through ctypes.  See the C file's
header for the passages of the RT-J int4 / int8 model cards each function
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, no FMA contraction)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call([
                "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm",
            ])
            os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_f16_from_double.restype = ctypes.c_uint16
        L.oracle_f16_from_double.argtypes = [ctypes.c_double]
        L.oracle_f16_to_double.restype = ctypes.c_double
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_pack_nibbles.argtypes = [_p, _i64, _p]
        L.oracle_unpack_nibbles.argtypes = [_p, _i64, _p]
        L.oracle_shrink_factor.restype = ctypes.c_double
        L.oracle_shrink_factor.argtypes = [ctypes.c_int, ctypes.c_int]
        L.oracle_q4_candidate.restype = ctypes.c_double
        L.oracle_q4_candidate.argtypes = [_p, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          _p, _p, _p]
        L.oracle_quant_q4_g32.restype = ctypes.c_int
        L.oracle_quant_q4_g32.argtypes = [_p, _i64, _i64, ctypes.c_int, _p, _p, _p]
        L.oracle_quant_q8_row.restype = ctypes.c_int
        L.oracle_quant_q8_row.argtypes = [_p, _i64, _i64, _p, _p]
        L.oracle_dequant_q4.argtypes = [_p, _p, _i64, _i64, _p]
        L.oracle_dequant_q8.argtypes = [_p, _p, _i64, _i64, _p]
        L.oracle_gemm_q4.restype = ctypes.c_int
        L.oracle_gemm_q4.argtypes = [_p, _p, _p, _i64, _i64, _i64, _p, _i64, _p, _p]
        L.oracle_gemm_q8.restype = ctypes.c_int
        L.oracle_gemm_q8.argtypes = [_p, _p, _p, _i64, _i64, _i64, _p, _i64, _p, _p]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_from_double.restype = ctypes.c_int
        L.oracle_e4m3_from_double.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_uint8)]
        L.oracle_quant_e4m3.restype = ctypes.c_int
        L.oracle_quant_e4m3.argtypes = [_p, _i64, _p]
        L.oracle_dequant_e4m3.argtypes = [_p, _i64, _i64, _p]
        L.oracle_gemm_e4m3.restype = ctypes.c_int
        L.oracle_gemm_e4m3.argtypes = [_p, _p, _i64, _i64, _i64, _p, _i64, _p, _p]
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# --------------------------------------------------------------------------
# fp16 helpers
# --------------------------------------------------------------------------
def f16_from_double(x: float) -> int:
    return int(lib().oracle_f16_from_double(float(x)))


def f16_to_double(h: int) -> float:
    return float(lib().oracle_f16_to_double(int(h) & 0xFFFF))


def shrink_factor(j: int, n_grid: int) -> float:
    return float(lib().oracle_shrink_factor(int(j), int(n_grid)))


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------
def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    assert codes.size % 2 == 0
    out = np.empty(codes.size // 2, dtype=np.uint8)
    lib().oracle_pack_nibbles(_ptr(codes), codes.size, _ptr(out))
    return out


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    lib().oracle_unpack_nibbles(_ptr(packed), out.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# quantizers
# --------------------------------------------------------------------------
def q4_candidate(w32: np.ndarray, lo: float, hi: float, s: float):
    """One grid point of the clip search: (scale16, min16, codes, err)."""
    w32 = np.ascontiguousarray(w32, dtype=np.float32)
    assert w32.size == 32
    sc = ctypes.c_uint16()
    mn = ctypes.c_uint16()
    codes = np.empty(32, dtype=np.uint8)
    err = lib().oracle_q4_candidate(_ptr(w32), lo, hi, s, ctypes.byref(sc), ctypes.byref(mn),
                                    _ptr(codes))
    return int(sc.value), int(mn.value), codes, float(err)


def quant_q4_g32(W: np.ndarray, n_grid: int = 21, want_j: bool = False):
    """Returns (Wq uint8 [N,K/2], scale_min uint16 [N,K/32,2][, jstar int32 [N,K/32]])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.empty((N, K // 2), dtype=np.uint8)
    sm = np.empty((N, K // 32, 2), dtype=np.uint16)
    js = np.empty((N, K // 32), dtype=np.int32)
    rc = lib().oracle_quant_q4_g32(_ptr(W), N, K, int(n_grid), _ptr(Wq), _ptr(sm), _ptr(js))
    if rc != 0:
        raise ValueError("oracle_quant_q4_g32 rejected its input")
    return (Wq, sm, js) if want_j else (Wq, sm)


def quant_q8_row(W: np.ndarray):
    """Returns (Wq int8 [N,K], scale float32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), dtype=np.int8)
    sc = np.empty((N,), dtype=np.float32)
    rc = lib().oracle_quant_q8_row(_ptr(W), N, K, _ptr(Wq), _ptr(sc))
    if rc != 0:
        raise ValueError("oracle_quant_q8_row rejected its input")
    return Wq, sc


# --------------------------------------------------------------------------
# dequantization and GEMM (double)
# --------------------------------------------------------------------------
def dequant_q4(Wq: np.ndarray, scale_min: np.ndarray) -> np.ndarray:
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    scale_min = np.ascontiguousarray(scale_min, dtype=np.uint16)
    N, K2 = Wq.shape
    out = np.empty((N, 2 * K2), dtype=np.float64)
    lib().oracle_dequant_q4(_ptr(Wq), _ptr(scale_min), N, 2 * K2, _ptr(out))
    return out


def dequant_q8(Wq: np.ndarray, scale: np.ndarray) -> np.ndarray:
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    N, K = Wq.shape
    out = np.empty((N, K), dtype=np.float64)
    lib().oracle_dequant_q8(_ptr(Wq), _ptr(scale), N, K, _ptr(out))
    return out


def _rows_arg(rows, M):
    if rows is None:
        return None, M
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < M))
    return rows, rows.size


def gemm_q4(X: np.ndarray, Wq: np.ndarray, scale_min: np.ndarray, rows=None) -> np.ndarray:
    """Y[r, o] = sum_k X[rows[r], k] * W_hat[o, k] in double (all rows when rows is None)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    scale_min = np.ascontiguousarray(scale_min, dtype=np.uint16)
    M, K = X.shape
    N = Wq.shape[0]
    assert Wq.shape == (N, K // 2) and scale_min.size == N * (K // 32) * 2
    rows, n = _rows_arg(rows, M)
    Y = np.empty((n, N), dtype=np.float64)
    wrow = np.empty(max(K, 1), dtype=np.float64)
    rc = lib().oracle_gemm_q4(_ptr(X), _ptr(Wq), _ptr(scale_min), M, N, K, _ptr(rows), n,
                              _ptr(Y), _ptr(wrow))
    if rc != 0:
        raise ValueError("oracle_gemm_q4: K must be a multiple of 32")
    return Y


def gemm_q8(X: np.ndarray, Wq: np.ndarray, scale: np.ndarray, rows=None) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.float32)
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M, K = X.shape
    N = Wq.shape[0]
    assert Wq.shape == (N, K) and scale.shape == (N,)
    rows, n = _rows_arg(rows, M)
    Y = np.empty((n, N), dtype=np.float64)
    wrow = np.empty(max(K, 1), dtype=np.float64)
    lib().oracle_gemm_q8(_ptr(X), _ptr(Wq), _ptr(scale), M, N, K, _ptr(rows), n,
                         _ptr(Y), _ptr(wrow))
    return Y


# --------------------------------------------------------------------------
# FP8 E4M3 (the FP8 card's float8_e4m3fn weights, no scale)
# --------------------------------------------------------------------------
def e4m3_to_double(b: int) -> float:
    return float(lib().oracle_e4m3_to_double(int(b) & 0xFF))


def e4m3_from_double(x: float):
    """Code of the nearest E4M3 value (ties to the even code); None if out of range."""
    out = ctypes.c_uint8()
    rc = lib().oracle_e4m3_from_double(float(x), ctypes.byref(out))
    return None if rc != 0 else int(out.value)


def quant_e4m3(W: np.ndarray) -> np.ndarray:
    """uint8 [N, K] of E4M3 codes; ValueError if a weight is out of range."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    out = np.empty(W.shape, dtype=np.uint8)
    if lib().oracle_quant_e4m3(_ptr(W), W.size, _ptr(out)) != 0:
        raise ValueError("oracle_quant_e4m3: a weight is NaN or beyond 464 in magnitude")
    return out


def dequant_e4m3(Wq: np.ndarray) -> np.ndarray:
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    N, K = Wq.shape
    out = np.empty((N, K), dtype=np.float64)
    lib().oracle_dequant_e4m3(_ptr(Wq), N, K, _ptr(out))
    return out


def gemm_e4m3(X: np.ndarray, Wq: np.ndarray, rows=None) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.float32)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    M, K = X.shape
    N = Wq.shape[0]
    assert Wq.shape == (N, K)
    rows, n = _rows_arg(rows, M)
    Y = np.empty((n, N), dtype=np.float64)
    wrow = np.empty(max(K, 1), dtype=np.float64)
    lib().oracle_gemm_e4m3(_ptr(X), _ptr(Wq), M, N, K, _ptr(rows), n, _ptr(Y), _ptr(wrow))
    return Y
