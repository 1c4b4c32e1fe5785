"""CPU oracle of the BitNet b1.58 BitLinear forward -- TEST INFRASTRUCTURE.

Only tests/, the package smoke check (__graft_entry__.smoke) and bench.py's
CPU-baseline / reference leg may import this module.  The product path (the
CUDA library and its Python binding) never touches it.

This is a thin numpy/ctypes wrapper around bitnet_oracle.c; every step of the
arithmetic, with its citation, is in that C file.  bf16 tensors travel as
numpy uint16 arrays holding the bf16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_rmsnorm_quant_act.argtypes = [P, ctypes.c_int, P, ctypes.c_float,
                                                 I64, I64, P, P, P, P]
        lib.oracle_weight_scale.argtypes = [P, I64, I64, P, P]
        lib.oracle_quantize_pack.argtypes = [P, I64, I64, ctypes.c_float, P, P]
        lib.oracle_unpack.argtypes = [P, I64, I64, P]
        lib.oracle_ternary_matmul_cols.argtypes = [P, P, I64, I64, I64, P, I64, P]
        lib.oracle_dequant.argtypes = [P, P, ctypes.c_float, I64, I64, P, P]
        lib.oracle_f32_to_bf16.argtypes = [P, P, I64]
        lib.oracle_f32_to_bf16.restype = None
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        for name in ("oracle_rmsnorm_quant_act", "oracle_weight_scale",
                     "oracle_quantize_pack", "oracle_unpack",
                     "oracle_ternary_matmul_cols", "oracle_dequant",
                     "oracle_set_threads"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def set_threads(n: int) -> int:
    """Threads used by the oracle's integer matmul; returns the count in effect."""
    return int(_load().oracle_set_threads(int(n)))


def _as_x(x):
    """Return (contiguous array, is_bf16) for fp32 or bf16-bits (uint16) input."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, 1
    if x.dtype == np.float32:
        return x, 0
    raise TypeError("x must be float32 or uint16 (bf16 bit patterns)")


def rmsnorm_quant_act(x, gamma=None, eps=1e-5):
    """RMSNorm + per-token absmax int8 quant.  x: [M,K] float32 or bf16 bits.
    Returns (x_q int8 [M,K], s_x float32 [M], rowsum int32 [M], x_n float32 [M,K])."""
    x, is_bf16 = _as_x(x)
    M, K = x.shape
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    x_q = np.empty((M, K), np.int8)
    s_x = np.empty((M,), np.float32)
    rs = np.empty((M,), np.int32)
    xn = np.empty((M, K), np.float32)
    _check(_load().oracle_rmsnorm_quant_act(_ptr(x), is_bf16, _ptr(g), float(eps), M, K,
                                            _ptr(x_q), _ptr(s_x), _ptr(xn), _ptr(rs)),
           "rmsnorm_quant_act")
    return x_q, s_x, rs, xn


def weight_scale(W):
    """Absmean per-tensor scale.  Returns (s_w float32 scalar, S = sum|W| fp64)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    s = np.empty((1,), np.float32)
    S = np.empty((1,), np.float64)
    _check(_load().oracle_weight_scale(_ptr(W), N, K, _ptr(s), _ptr(S)), "weight_scale")
    return np.float32(s[0]), float(S[0])


def quantize_pack(W, s_w):
    """Ternarize with scale s_w and pack.  Returns (W_p uint8 [N,K/4], T int8 [N,K])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    W_p = np.empty((N, K // 4), np.uint8)
    T = np.empty((N, K), np.int8)
    _check(_load().oracle_quantize_pack(_ptr(W), N, K, float(np.float32(s_w)),
                                        _ptr(W_p), _ptr(T)), "quantize_pack")
    return W_p, T


def unpack(W_p, K):
    """Packed bytes [N,K/4] -> ternary int8 [N,K]."""
    W_p = np.ascontiguousarray(W_p, dtype=np.uint8)
    N = W_p.shape[0]
    T = np.empty((N, K), np.int8)
    _check(_load().oracle_unpack(_ptr(W_p), N, K, _ptr(T)), "unpack")
    return T


def ternary_matmul(x_q, W_p, K, cols=None):
    """acc[m, c] = sum_k x_q[m,k] * T[cols[c],k]  (int32).  cols None = all rows of W_p."""
    x_q = np.ascontiguousarray(x_q, dtype=np.int8)
    W_p = np.ascontiguousarray(W_p, dtype=np.uint8)
    M = x_q.shape[0]
    N = W_p.shape[0]
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = N if c is None else c.shape[0]
    acc = np.empty((M, nc), np.int32)
    _check(_load().oracle_ternary_matmul_cols(_ptr(x_q), _ptr(W_p), M, N, K, _ptr(c), nc,
                                              _ptr(acc)), "ternary_matmul")
    return acc


def dequant(acc, s_x, s_w):
    """y = acc / (s_x[m] * s_w).  Returns (y float32, y_bf16 uint16 bits)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    M, nc = acc.shape
    y = np.empty((M, nc), np.float32)
    yb = np.empty((M, nc), np.uint16)
    _check(_load().oracle_dequant(_ptr(acc), _ptr(s_x), float(np.float32(s_w)), M, nc,
                                  _ptr(y), _ptr(yb)), "dequant")
    return y, yb


def f32_to_bf16(a):
    """fp32 array -> bf16 bit patterns (round to nearest even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().oracle_f32_to_bf16(_ptr(a), _ptr(out), a.size)
    return out


def linear_forward(x, gamma, eps, W_p, s_w, K, cols=None):
    """Whole BitLinear forward for output columns `cols` (None = all).
    Returns dict with x_q, s_x, rowsum, acc, y (fp32), y_bf16 (bits)."""
    x_q, s_x, rowsum, _ = rmsnorm_quant_act(x, gamma, eps)
    acc = ternary_matmul(x_q, W_p, K, cols)
    y, yb = dequant(acc, s_x, s_w)
    return {"x_q": x_q, "s_x": s_x, "rowsum": rowsum, "acc": acc, "y": y, "y_bf16": yb}


def bf16_bits_to_f32(bits):
    """bf16 bit patterns -> float32 (exact widening)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


__all__ = ["set_threads", "rmsnorm_quant_act", "weight_scale", "quantize_pack", "unpack",
           "ternary_matmul", "dequant", "f32_to_bf16", "linear_forward", "bf16_bits_to_f32"]
