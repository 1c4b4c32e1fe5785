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


# ------------------------------------------------------------ forward variants

def _load_variants():
    lib = _load()
    if getattr(lib, "_variants", False):
        return lib
    P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    lib.oracle_swiglu.argtypes = [P, P, I64, P, P]
    lib.oracle_warmup_forward.argtypes = [P, ctypes.c_int, P, F, P, I64, I64, I64, F, P, I64,
                                          P, P, P, P]
    lib.oracle_bitdelta_compress.argtypes = [P, P, I64, I64, P, P, P]
    lib.oracle_bitdelta_forward.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P, P]
    lib.oracle_group_weight_scale.argtypes = [P, I64, I64, I64, P]
    lib.oracle_group_quantize_pack.argtypes = [P, I64, I64, I64, P, P]
    lib.oracle_group_rmsnorm_quant_act.argtypes = [P, ctypes.c_int, P, F, I64, I64, I64, P, P]
    lib.oracle_group_matmul_dequant.argtypes = [P, P, P, P, I64, I64, I64, I64, P, I64, P, P, P]
    lib.oracle_warmup_weights.argtypes = [P, I64, I64, F, P, P]
    for name in ("oracle_swiglu", "oracle_warmup_forward", "oracle_warmup_weights",
                 "oracle_bitdelta_compress",
                 "oracle_bitdelta_forward", "oracle_group_weight_scale",
                 "oracle_group_quantize_pack", "oracle_group_rmsnorm_quant_act",
                 "oracle_group_matmul_dequant"):
        getattr(lib, name).restype = ctypes.c_int
    lib._variants = True
    return lib


def swiglu(g, u):
    """silu(g) * u from two fp32 arrays.  Returns (fp32, bf16 bits)."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    u = np.ascontiguousarray(u, dtype=np.float32)
    if g.shape != u.shape:
        raise ValueError("g and u must have the same shape")
    o = np.empty(g.shape, np.float32)
    ob = np.empty(g.shape, np.uint16)
    _check(_load_variants().oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(o), _ptr(ob)),
           "swiglu")
    return o, ob


def swiglu_forward(x, gamma, eps, Wg_p, s_wg, Wu_p, s_wu, K, cols=None):
    """The SwiGLU of two BitLinear forwards of the same input x: silu(gate) * up."""
    g = linear_forward(x, gamma, eps, Wg_p, s_wg, K, cols)
    u = linear_forward(x, gamma, eps, Wu_p, s_wu, K, cols)
    y, yb = swiglu(g["y"], u["y"])
    return {"gate": g, "up": u, "y": y, "y_bf16": yb}


def warmup_lambda(step, total_steps):
    """The warm-up weight of the quantization: min(step / total_steps, 1)."""
    if total_steps <= 0:
        raise ValueError("total_steps must be positive")
    return min(float(step) / float(total_steps), 1.0)


def warmup_forward(x, gamma, eps, W, lam, cols=None):
    """The lambda-warmup fake-quant forward.  Returns dict with y (fp64 on the
    fp32 operands), y_b (fp64 on their bf16 roundings), absdot, x_lam."""
    x, is_bf16 = _as_x(x)
    W = np.ascontiguousarray(W, dtype=np.float32)
    M, K = x.shape
    N = W.shape[0]
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = N if c is None else c.shape[0]
    y = np.empty((M, nc), np.float64)
    yb = np.empty((M, nc), np.float64)
    ad = np.empty((M, nc), np.float64)
    xl = np.empty((M, K), np.float32)
    _check(_load_variants().oracle_warmup_forward(
        _ptr(x), is_bf16, _ptr(g), float(eps), _ptr(W), M, N, K, float(np.float32(lam)),
        _ptr(c), nc, _ptr(xl), _ptr(y), _ptr(yb), _ptr(ad)), "warmup_forward")
    return {"y": y, "y_b": yb, "absdot": ad, "x_lam": xl}


def warmup_weights(W, lam):
    """(W_lam fp32 [N,K], s_w): the weight operand of the warm-up forward."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    out = np.empty((N, K), np.float32)
    s = np.empty((1,), np.float32)
    _check(_load_variants().oracle_warmup_weights(_ptr(W), N, K, float(np.float32(lam)),
                                                  _ptr(out), _ptr(s)), "warmup_weights")
    return out, np.float32(s[0])


def warmup_backward(dy_bits, x_lam_bits, W_lam_bits):
    """Straight-through backward of y = x_lam W_lam^T (the warm-up page's
    estimator: the quantizers pass the gradient through unchanged), on bf16
    operands given as bit patterns: dx = dy W_lam, dW = dy^T x_lam, each a
    plain matrix product of the exactly widened values summed in fp64."""
    dy = bf16_bits_to_f32(dy_bits).astype(np.float64)
    xl = bf16_bits_to_f32(x_lam_bits).astype(np.float64)
    wl = bf16_bits_to_f32(W_lam_bits).astype(np.float64)
    return dy @ wl, dy.T @ xl


def bitdelta_compress(W_base_bits, W_fine_bits):
    """Sign bits [N, K/32] (uint32) and alpha (fp32) of W_fine - W_base (bf16 bits)."""
    Wb = np.ascontiguousarray(W_base_bits, dtype=np.uint16)
    Wf = np.ascontiguousarray(W_fine_bits, dtype=np.uint16)
    N, K = Wb.shape
    signs = np.empty((N, K // 32), np.uint32)
    a = np.empty((1,), np.float32)
    S = np.empty((1,), np.float64)
    _check(_load_variants().oracle_bitdelta_compress(_ptr(Wb), _ptr(Wf), N, K, _ptr(signs),
                                                     _ptr(a), _ptr(S)), "bitdelta_compress")
    return signs, np.float32(a[0]), float(S[0])


def bitdelta_forward(x_bits, W_base_bits, signs, alpha, cols=None):
    """y [B, ncols] (fp64) and absdot for B tenants: x_bits [B, K], signs [B, N, K/32]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    Wb = np.ascontiguousarray(W_base_bits, dtype=np.uint16)
    sg = np.ascontiguousarray(signs, dtype=np.uint32)
    al = np.ascontiguousarray(alpha, dtype=np.float32)
    B, K = x.shape
    N = Wb.shape[0]
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = N if c is None else c.shape[0]
    y = np.empty((B, nc), np.float64)
    ad = np.empty((B, nc), np.float64)
    _check(_load_variants().oracle_bitdelta_forward(_ptr(x), _ptr(Wb), _ptr(sg), _ptr(al), B, N,
                                                    K, _ptr(c), nc, _ptr(y), _ptr(ad)),
           "bitdelta_forward")
    return y, ad


def group_weight_scale(W, group_k):
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    s = np.empty((K // group_k,), np.float32)
    _check(_load_variants().oracle_group_weight_scale(_ptr(W), N, K, int(group_k), _ptr(s)),
           "group_weight_scale")
    return s


def group_quantize_pack(W, group_k, s_w):
    W = np.ascontiguousarray(W, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    N, K = W.shape
    W_p = np.empty((N, K // 4), np.uint8)
    _check(_load_variants().oracle_group_quantize_pack(_ptr(W), N, K, int(group_k), _ptr(s_w),
                                                       _ptr(W_p)), "group_quantize_pack")
    return W_p


def group_rmsnorm_quant_act(x, gamma, eps, group_k):
    x, is_bf16 = _as_x(x)
    M, K = x.shape
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    x_q = np.empty((M, K), np.int8)
    s_x = np.empty((M, K // group_k), np.float32)
    _check(_load_variants().oracle_group_rmsnorm_quant_act(_ptr(x), is_bf16, _ptr(g),
                                                           float(eps), M, K, int(group_k),
                                                           _ptr(x_q), _ptr(s_x)),
           "group_rmsnorm_quant_act")
    return x_q, s_x


def group_linear_forward(x, gamma, eps, W_p, s_w, K, group_k, cols=None):
    """The group-scale forward.  Returns dict with x_q, s_x [M,G], acc [M,ncols,G],
    y (fp32), y_bf16."""
    x_q, s_x = group_rmsnorm_quant_act(x, gamma, eps, group_k)
    W_p = np.ascontiguousarray(W_p, dtype=np.uint8)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M = x_q.shape[0]
    N = W_p.shape[0]
    G = K // group_k
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nc = N if c is None else c.shape[0]
    acc = np.empty((M, nc, G), np.int32)
    y = np.empty((M, nc), np.float32)
    yb = np.empty((M, nc), np.uint16)
    _check(_load_variants().oracle_group_matmul_dequant(
        _ptr(x_q), _ptr(s_x), _ptr(W_p), _ptr(s_w), M, N, K, int(group_k), _ptr(c), nc,
        _ptr(acc), _ptr(y), _ptr(yb)), "group_matmul_dequant")
    return {"x_q": x_q, "s_x": s_x, "acc": acc, "y": y, "y_bf16": yb}


__all__ += ["swiglu", "swiglu_forward", "warmup_lambda", "warmup_forward", "warmup_weights",
            "warmup_backward",
            "bitdelta_compress", "bitdelta_forward", "group_weight_scale",
            "group_quantize_pack", "group_rmsnorm_quant_act", "group_linear_forward"]
