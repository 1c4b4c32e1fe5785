"""B200 (sm_100a) BitNet b1.58 BitLinear forward -- Python binding.

Thin ctypes marshalling over libbitnet_b200.so: the functions below carry the
names of the C entry points declared in include/bitnet_b200.h, take torch
CUDA tensors, check dtypes/shapes, and pass raw device pointers plus the
current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; PyTorch only provides device memory and streams.  There is no
CPU fallback: if the library is missing or a call fails, an exception is
raised.
"""
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_UNSUPPORTED_SHAPE = 2
BITNET_ERR_MISALIGNED = 3
BITNET_ERR_CUDA = 4
BITNET_ERR_TIMEOUT = 5
BITNET_ERR_WORKSPACE = 6
BITNET_ERR_SCRATCH_LIMIT = 7
BITNET_STATIC_SCRATCH_MAX_N = 65536
BITNET_MAX_K = 1 << 20
BITNET_MAX_M = 65535 * 128
BITNET_MAX_N = 1 << 24

BITNET_F32 = 0
BITNET_BF16 = 1

BITNET_PATH_AUTO = 0
BITNET_PATH_GEMV = 1
BITNET_PATH_GEMM = 2

# Every entry point the header declares (checked by the tests).
EXPORTED = (
    "bitnet_status_string", "bitnet_version",
    "bitnet_quantize_pack_weights_workspace_bytes", "bitnet_quantize_pack_weights",
    "bitnet_rmsnorm_quant_act", "bitnet_linear_forward_workspace_bytes",
    "bitnet_linear_forward", "bitnet_linear_quantize_input", "bitnet_linear_matmul",
    "bitnet_linear_forward_debug", "bitnet_ternary_matmul_i32",
    "bitnet_device_status", "bitnet_selftest_bounded_wait", "bitnet_selftest_divide",
    "bitnet_quantize_pack_weights_static",
    "bitnet_linear_forward_grouped_workspace_bytes", "bitnet_linear_forward_grouped",
    "bitnet_workspace_bytes", "bitnet_last_device_status",
    "bitnet_tiled_weights_bytes", "bitnet_tile_weights", "bitnet_linear_forward_ex",
    "bitnet_selftest_mma_i8",
    "bitnet_tiled_pair_weights_bytes", "bitnet_tile_weights_pair",
    "bitnet_swiglu_forward_workspace_bytes", "bitnet_swiglu_forward",
    "bitnet_last_cuda_error",
    "bitnet_quantize_pack_weights_group_scales_workspace_bytes",
    "bitnet_quantize_pack_weights_group_scales",
    "bitnet_linear_forward_group_scales_workspace_bytes", "bitnet_linear_forward_group_scales",
    "bitnet_warmup_quantize_weights_workspace_bytes", "bitnet_warmup_quantize_weights",
    "bitnet_warmup_forward_workspace_bytes", "bitnet_warmup_forward",
    "bitnet_warmup_backward_workspace_bytes", "bitnet_warmup_backward",
    "bitnet_bitdelta_compress_workspace_bytes", "bitnet_bitdelta_compress",
    "bitnet_bitdelta_forward",
)

BITNET_LAYOUT_ROWS = 0
BITNET_LAYOUT_TILED = 1

BITNET_MAX_GROUP = 16
BITNET_PHASE_QUANTIZE = 1
BITNET_PHASE_MATMUL = 2
BITNET_PHASE_ALL = 3


class LinearProblem(ctypes.Structure):
    """Mirror of bitnet_linear_problem (include/bitnet_b200.h)."""
    _fields_ = [("x", ctypes.c_void_p), ("x_dtype", ctypes.c_int),
                ("gamma", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("W_packed", ctypes.c_void_p), ("s_w", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("y", ctypes.c_void_p), ("y_dtype", ctypes.c_int), ("w_layout", ctypes.c_int)]


class BitnetError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed: {msg} (status {code})")
        self.code = code


_lib = None
_lib_lock = threading.Lock()


def load_library(path: str = LIB_PATH):
    """Load (once) and return the ctypes handle of libbitnet_b200.so."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing; build it with `python ternary_quantized_linear_b200/build.py`"
                " (there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        F = ctypes.c_float
        sig = {
            "bitnet_status_string": ([I], ctypes.c_char_p),
            "bitnet_version": ([], I),
            "bitnet_quantize_pack_weights_workspace_bytes": ([I64, I64], SZ),
            "bitnet_quantize_pack_weights": ([P, I64, I64, P, P, P, SZ, P], I),
            "bitnet_rmsnorm_quant_act": ([P, I, P, F, I64, I64, P, P, P], I),
            "bitnet_linear_forward_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_linear_forward": ([P, I, P, F, P, P, I64, I64, I64, P, I, P, SZ, P], I),
            "bitnet_linear_quantize_input": ([P, I, P, F, I64, I64, I64, P, SZ, P], I),
            "bitnet_linear_matmul": ([P, P, I64, I64, I64, P, I, P, SZ, P], I),
            "bitnet_linear_forward_debug": (
                [P, I, P, F, P, P, I64, I64, I64, P, I, P, SZ, P, P, P, I, P], I),
            "bitnet_ternary_matmul_i32": ([P, P, I64, I64, I64, P, P, SZ, I, P], I),
            "bitnet_device_status": ([P, I, ctypes.POINTER(I)], I),
            "bitnet_selftest_bounded_wait": ([ctypes.c_uint64, P], I),
            "bitnet_selftest_divide": ([P, P, P, I64, P], I),
            "bitnet_quantize_pack_weights_static": ([P, I64, I64, P, P, P], I),
            "bitnet_linear_forward_grouped_workspace_bytes": ([I, P], SZ),
            "bitnet_linear_forward_grouped": ([I, P, P, SZ, I, P], I),
            "bitnet_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_last_device_status": ([P], I),
            "bitnet_tiled_weights_bytes": ([I64, I64], SZ),
            "bitnet_tile_weights": ([P, I64, I64, P, P], I),
            "bitnet_linear_forward_ex": ([P, P, SZ, P, P, P, I, P], I),
            "bitnet_selftest_mma_i8": ([I64, I, I, P], I),
            "bitnet_tiled_pair_weights_bytes": ([I64, I64], SZ),
            "bitnet_tile_weights_pair": ([P, P, I64, I64, P, P], I),
            "bitnet_swiglu_forward_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_swiglu_forward": ([P, I, P, F, P, P, P, I64, I64, I64, P, I, P, SZ, P], I),
            "bitnet_last_cuda_error": ([ctypes.POINTER(ctypes.c_char_p)], I),
            "bitnet_quantize_pack_weights_group_scales_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_quantize_pack_weights_group_scales": ([P, I64, I64, I64, P, P, P, SZ, P], I),
            "bitnet_linear_forward_group_scales_workspace_bytes": ([I64, I64, I64, I64], SZ),
            "bitnet_linear_forward_group_scales": (
                [P, I, P, F, P, I, P, I64, I64, I64, I64, P, I, P, SZ, P, P, P, P], I),
            "bitnet_warmup_quantize_weights_workspace_bytes": ([I64, I64], SZ),
            "bitnet_warmup_quantize_weights": ([P, I64, I64, F, P, P, P, SZ, P], I),
            "bitnet_warmup_forward_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_warmup_forward": ([P, I, P, F, P, I64, I64, I64, F, P, I, P, P, SZ, P], I),
            "bitnet_warmup_backward_workspace_bytes": ([I64, I64, I64], SZ),
            "bitnet_warmup_backward": ([P, P, P, I64, I64, I64, P, P, P, SZ, P], I),
            "bitnet_bitdelta_compress_workspace_bytes": ([I64, I64], SZ),
            "bitnet_bitdelta_compress": ([P, P, I64, I64, P, P, P, SZ, P], I),
            "bitnet_bitdelta_forward": ([P, P, P, P, I64, I64, I64, P, I, P], I),
        }
        for name, (argtypes, restype) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = restype
        _lib = lib
        return lib


def _check(fn_name, code):
    if code != BITNET_OK:
        lib = load_library()
        msg = lib.bitnet_status_string(code).decode()
        if code == BITNET_ERR_CUDA:
            name = ctypes.c_char_p()
            err = lib.bitnet_last_cuda_error(ctypes.byref(name))
            if err:
                msg += f" ({name.value.decode() if name.value else 'cudaError'} = {err})"
        raise BitnetError(fn_name, code, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt):
    if dt == torch.float32:
        return BITNET_F32
    if dt == torch.bfloat16:
        return BITNET_BF16
    raise TypeError(f"unsupported dtype {dt} (float32 or bfloat16)")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _expect(t, name, dtypes, numel=None, shape=None):
    """Check a caller-supplied buffer before its pointer reaches the library,
    which cannot see sizes or element types: a wrong dtype or a buffer too
    small for what the call writes raises here instead of becoming an
    out-of-range device access."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not isinstance(dtypes, tuple):
        dtypes = (dtypes,)
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}, "
                        f"got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {numel}")


def _expect_gamma(gamma, K):
    if gamma is not None:
        _expect(gamma, "gamma", torch.float32, shape=(K,))


def _expect_x(x):
    if x.dim() != 2:
        raise ValueError("x must be 2-D [M, K]")
    _expect(x, "x", (torch.float32, torch.bfloat16))
    return x.shape


def _expect_packed(W_packed, K=None):
    _expect(W_packed, "W_packed", torch.uint8)
    if W_packed.dim() != 2 or (K is not None and W_packed.shape[1] * 4 != K):
        raise ValueError("W_packed must be uint8 [N, K/4]")
    return W_packed.shape[0]


class Workspace:
    """Device scratch reused across stream-ordered calls (one buffer per
    device and stream, grown on demand; the library clears what it needs)."""

    def __init__(self):
        self._buf = {}

    def get(self, nbytes, device, stream=None):
        # Key on the stream the call will actually run on (the current one
        # when none is given): two streams must never share a buffer.
        dev = torch.device("cuda", device.index if isinstance(device, torch.device)
                           else int(device))
        s = torch.cuda.current_stream(dev) if stream is None else stream
        key = (dev.index, s.cuda_stream)
        buf = self._buf.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
            self._buf[key] = buf
        return buf


_default_ws = Workspace()


def bitnet_version() -> int:
    return int(load_library().bitnet_version())


def bitnet_status_string(code: int) -> str:
    return load_library().bitnet_status_string(int(code)).decode()


def bitnet_quantize_pack_weights_workspace_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_quantize_pack_weights_workspace_bytes(N, K))


def bitnet_linear_forward_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load_library().bitnet_linear_forward_workspace_bytes(M, N, K))


def _expect_weights(W):
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, K]")
    _expect(W, "W", torch.float32)
    return W.shape


def bitnet_quantize_pack_weights(W, W_packed=None, s_w=None, workspace=None, stream=None):
    """W fp32 [N,K] -> (W_packed uint8 [N,K/4], s_w fp32 [1]) on W's device."""
    N, K = _expect_weights(W)
    if W_packed is not None:
        _expect(W_packed, "W_packed", torch.uint8, numel=N * (K // 4))
    if s_w is not None:
        _expect(s_w, "s_w", torch.float32, numel=1)
    nb = bitnet_quantize_pack_weights_workspace_bytes(N, K)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(W, W_packed, s_w, workspace)
    if W_packed is None:
        W_packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if s_w is None:
        s_w = torch.empty((1,), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=W.device)
    _check("bitnet_quantize_pack_weights", load_library().bitnet_quantize_pack_weights(
        _ptr(W), N, K, _ptr(W_packed), _ptr(s_w), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return W_packed, s_w


def bitnet_quantize_pack_weights_static(W, W_packed, s_w, stream=None):
    """Weight quantization + packing that allocates nothing: for callers that
    cannot allocate device memory (e.g. plugins of an engine that owns the
    memory budget).  The caller provides W, W_packed [N,K/4] and s_w [1]; the
    library's own static scratch (N <= 65536 rows) replaces the workspace.
    Calls on one device share that scratch, so calls that overlap on the GPU
    race."""
    N, K = _expect_weights(W)
    _expect(W_packed, "W_packed", torch.uint8, numel=N * (K // 4))
    _expect(s_w, "s_w", torch.float32, numel=1)
    _need_cuda(W, W_packed, s_w)
    _check("bitnet_quantize_pack_weights_static",
           load_library().bitnet_quantize_pack_weights_static(
               _ptr(W), N, K, _ptr(W_packed), _ptr(s_w), _stream(stream)))
    return W_packed, s_w


def bitnet_rmsnorm_quant_act(x, gamma=None, eps=1e-5, x_q=None, s_x=None, stream=None):
    """x [M,K] fp32/bf16 -> (x_q int8 [M,K], s_x fp32 [M])."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    if x_q is not None:
        _expect(x_q, "x_q", torch.int8, numel=M * K)
    if s_x is not None:
        _expect(s_x, "s_x", torch.float32, numel=M)
    _need_cuda(x, gamma, x_q, s_x)
    if x_q is None:
        x_q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if s_x is None:
        s_x = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("bitnet_rmsnorm_quant_act", load_library().bitnet_rmsnorm_quant_act(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), M, K, _ptr(x_q), _ptr(s_x),
        _stream(stream)))
    return x_q, s_x


def _ws_for(M, N, K, device, workspace, stream):
    nb = bitnet_linear_forward_workspace_bytes(M, N, K)
    if workspace is None:
        workspace = _default_ws.get(nb, device, stream)
    _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(workspace)
    return workspace


def _expect_y(y, M, N, dtypes=(torch.float32, torch.bfloat16)):
    _expect(y, "y", dtypes, numel=M * N)
    if y.dim() != 2 or tuple(y.shape) != (M, N):
        raise ValueError(f"y must have shape ({M}, {N}), got {tuple(y.shape)}")


def _expect_scale(s_w):
    _expect(s_w, "s_w", torch.float32, numel=1)


def bitnet_linear_forward(x, gamma, eps, W_packed, s_w, y_dtype=torch.bfloat16, y=None,
                          workspace=None, stream=None):
    """y = BitLinear(x) with packed ternary weights; y [M,N] in y_dtype."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    N = _expect_packed(W_packed, K)
    _expect_scale(s_w)
    if y is not None:
        _expect_y(y, M, N)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8,
                numel=bitnet_linear_forward_workspace_bytes(M, N, K))
    _need_cuda(x, gamma, W_packed, s_w, y, workspace)
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    ws = _ws_for(M, N, K, x.device, workspace, stream)
    _check("bitnet_linear_forward", load_library().bitnet_linear_forward(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), _ptr(W_packed), _ptr(s_w),
        M, N, K, _ptr(y), _dtype_code(y.dtype), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def bitnet_linear_quantize_input(x, gamma, eps, N, workspace, stream=None):
    """Phase 1 of the forward: quantize x [M,K] into `workspace` (sized for (M,N,K))."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    _expect(workspace, "workspace", torch.uint8,
            numel=bitnet_linear_forward_workspace_bytes(M, int(N), K))
    _need_cuda(x, gamma, workspace)
    _check("bitnet_linear_quantize_input", load_library().bitnet_linear_quantize_input(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), M, int(N), K, _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return workspace


def bitnet_linear_matmul(W_packed, s_w, M, K, workspace, y_dtype=torch.bfloat16, y=None,
                         stream=None):
    """Phase 2: y [M,N] = dequant(quantized input in `workspace` x ternary(W)^T)."""
    M, K = int(M), int(K)
    N = _expect_packed(W_packed, K)
    _expect_scale(s_w)
    _expect(workspace, "workspace", torch.uint8,
            numel=bitnet_linear_forward_workspace_bytes(M, N, K))
    if y is not None:
        _expect_y(y, M, N)
    _need_cuda(W_packed, s_w, workspace, y)
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=W_packed.device)
    _check("bitnet_linear_matmul", load_library().bitnet_linear_matmul(
        _ptr(W_packed), _ptr(s_w), M, N, K, _ptr(y), _dtype_code(y.dtype),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return y


class TiledWeights:
    """Packed weights in the tiled layout (bitnet_tile_weights): the flat byte
    buffer plus the matrix shape it holds."""

    def __init__(self, data, N, K):
        _expect(data, "tiled weights", torch.uint8,
                numel=bitnet_tiled_weights_bytes(int(N), int(K)))
        self.data, self.N, self.K = data, int(N), int(K)
        self.shape = (self.N, self.K // 4)

    @property
    def device(self):
        return self.data.device


def bitnet_tiled_weights_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_tiled_weights_bytes(int(N), int(K)))


def bitnet_tile_weights(W_packed, out=None, stream=None):
    """Row-major packed weights uint8 [N, K/4] -> TiledWeights (same codes,
    in the tiled order the matmul kernels stream fastest)."""
    N = _expect_packed(W_packed)
    K = W_packed.shape[1] * 4
    nb = bitnet_tiled_weights_bytes(N, K)
    if nb == 0:
        raise ValueError(f"unsupported shape N={N}, K={K}")
    if out is not None:
        _expect(out, "out", torch.uint8, numel=nb)
    _need_cuda(W_packed, out)
    if out is None:
        out = torch.empty(nb, dtype=torch.uint8, device=W_packed.device)
    _check("bitnet_tile_weights", load_library().bitnet_tile_weights(
        _ptr(W_packed), N, K, _ptr(out), _stream(stream)))
    return TiledWeights(out, N, K)


class PairTiledWeights:
    """The gate and up projections of a SwiGLU in the pair-tiled layout
    (bitnet_tile_weights_pair): flat bytes plus the shape of each matrix."""

    def __init__(self, data, N, K):
        _expect(data, "pair-tiled weights", torch.uint8,
                numel=bitnet_tiled_pair_weights_bytes(int(N), int(K)))
        self.data, self.N, self.K = data, int(N), int(K)
        self.shape = (self.N, self.K // 4)


def bitnet_tiled_pair_weights_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_tiled_pair_weights_bytes(int(N), int(K)))


def bitnet_tile_weights_pair(W_gate, W_up, out=None, stream=None):
    """Two row-major packed matrices of the same shape [N, K/4] -> their
    pair-tiled layout (for bitnet_swiglu_forward)."""
    N = _expect_packed(W_gate)
    K = W_gate.shape[1] * 4
    if tuple(W_up.shape) != tuple(W_gate.shape):
        raise ValueError("W_gate and W_up must have the same shape")
    _expect_packed(W_up, K)
    nb = bitnet_tiled_pair_weights_bytes(N, K)
    if nb == 0:
        raise ValueError(f"unsupported shape N={N}, K={K}")
    if out is not None:
        _expect(out, "out", torch.uint8, numel=nb)
    _need_cuda(W_gate, W_up, out)
    if out is None:
        out = torch.empty(nb, dtype=torch.uint8, device=W_gate.device)
    _check("bitnet_tile_weights_pair", load_library().bitnet_tile_weights_pair(
        _ptr(W_gate), _ptr(W_up), N, K, _ptr(out), _stream(stream)))
    return PairTiledWeights(out, N, K)


def bitnet_swiglu_forward(x, gamma, eps, W_pair, s_w_gate, s_w_up, y_dtype=torch.bfloat16,
                          y=None, workspace=None, stream=None):
    """silu(gate) * up of the two BitLinear forwards of x (M <= 16 tokens),
    fused into one decode matmul launch.  W_pair: PairTiledWeights."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    if not isinstance(W_pair, PairTiledWeights) or W_pair.K != K:
        raise ValueError("W_pair must be PairTiledWeights with the input's K")
    N = W_pair.N
    _expect_scale(s_w_gate)
    _expect_scale(s_w_up)
    if y is not None:
        _expect_y(y, M, N)
    nb = int(load_library().bitnet_swiglu_forward_workspace_bytes(M, N, K))
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(x, gamma, W_pair.data, s_w_gate, s_w_up, y, workspace)
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    if workspace is None:
        workspace = _default_ws.get(nb, x.device, stream)
    _check("bitnet_swiglu_forward", load_library().bitnet_swiglu_forward(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), _ptr(W_pair.data),
        _ptr(s_w_gate), _ptr(s_w_up), M, N, K, _ptr(y), _dtype_code(y.dtype), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return y


def bitnet_quantize_pack_weights_group_scales(W, group_k, W_packed=None, s_w=None,
                                              workspace=None, stream=None):
    """W fp32 [N,K] -> (W_packed uint8 [N,K/4], s_w fp32 [K/group_k]): one
    absmean scale per group of group_k consecutive input features."""
    N, K = _expect_weights(W)
    group_k = int(group_k)
    if group_k <= 0 or K % group_k:
        raise ValueError("group_k must divide K")
    G = K // group_k
    if W_packed is not None:
        _expect(W_packed, "W_packed", torch.uint8, numel=N * (K // 4))
    if s_w is not None:
        _expect(s_w, "s_w", torch.float32, numel=G)
    lib = load_library()
    nb = int(lib.bitnet_quantize_pack_weights_group_scales_workspace_bytes(N, K, group_k))
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(W, W_packed, s_w, workspace)
    if W_packed is None:
        W_packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if s_w is None:
        s_w = torch.empty((G,), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=W.device)
    _check("bitnet_quantize_pack_weights_group_scales",
           lib.bitnet_quantize_pack_weights_group_scales(
               _ptr(W), N, K, group_k, _ptr(W_packed), _ptr(s_w), _ptr(workspace),
               workspace.numel(), _stream(stream)))
    return W_packed, s_w


def bitnet_linear_forward_group_scales(x, gamma, eps, W, s_w, group_k, y_dtype=torch.float32,
                                       y=None, debug=False, workspace=None, stream=None):
    """The forward with group-wise scales (W row-major [N, K/4] or
    TiledWeights, s_w [K/group_k]).  With debug, also returns x_q (natural
    order), s_x [M, G] and the per-group integer sums acc [G, M, N]."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    group_k = int(group_k)
    if group_k <= 0 or K % group_k:
        raise ValueError("group_k must divide K")
    G = K // group_k
    if not isinstance(W, TiledWeights):
        _expect_packed(W, K)
    N = W.shape[0]
    _expect(s_w, "s_w", torch.float32, numel=G)
    if y is not None:
        _expect_y(y, M, N)
    lib = load_library()
    nb = int(lib.bitnet_linear_forward_group_scales_workspace_bytes(M, N, K, group_k))
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(x, gamma, s_w, y, workspace)
    wp, layout, _ = _weights_ptr_layout(W, K)
    dev = x.device
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=dev)
    x_q = torch.empty((M, K), dtype=torch.int8, device=dev) if debug else None
    s_x = torch.empty((M, G), dtype=torch.float32, device=dev) if debug else None
    acc = torch.empty((G, M, N), dtype=torch.int32, device=dev) if debug else None
    if workspace is None:
        workspace = _default_ws.get(nb, dev, stream)
    _check("bitnet_linear_forward_group_scales", lib.bitnet_linear_forward_group_scales(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), ctypes.c_void_p(wp), layout,
        _ptr(s_w), M, N, K, group_k, _ptr(y), _dtype_code(y.dtype), _ptr(workspace),
        workspace.numel(), _ptr(x_q), _ptr(s_x), _ptr(acc), _stream(stream)))
    return {"y": y, "x_q": x_q, "s_x": s_x, "acc": acc}


def _check_lambda(lam):
    lam = float(lam)
    if not (0.0 <= lam <= 1.0):
        raise ValueError("lambda must be in [0, 1]")
    return lam


def bitnet_warmup_quantize_weights(W, lam, W_lam=None, s_w=None, workspace=None, stream=None):
    """W fp32 [N,K] -> (W_lam bf16 [N,K], s_w fp32 [1]): the warm-up blend
    W + lam (t / s_w - W) of the weights, rounded to bf16."""
    N, K = _expect_weights(W)
    lam = _check_lambda(lam)
    if W_lam is not None:
        _expect(W_lam, "W_lam", torch.bfloat16, shape=(N, K))
    if s_w is not None:
        _expect(s_w, "s_w", torch.float32, numel=1)
    lib = load_library()
    nb = int(lib.bitnet_warmup_quantize_weights_workspace_bytes(N, K))
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(W, W_lam, s_w, workspace)
    if W_lam is None:
        W_lam = torch.empty((N, K), dtype=torch.bfloat16, device=W.device)
    if s_w is None:
        s_w = torch.empty((1,), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=W.device)
    _check("bitnet_warmup_quantize_weights", lib.bitnet_warmup_quantize_weights(
        _ptr(W), N, K, ctypes.c_float(lam), _ptr(W_lam), _ptr(s_w), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return W_lam, s_w


def bitnet_warmup_forward(x, gamma, eps, W_lam, lam, y_dtype=torch.float32, y=None,
                          keep_x_lam=False, stream=None):
    """y = x_lam W_lam^T with x_lam = x_n + lam (x_q / s_x - x_n) (bf16 tensor
    cores, fp32 sums).  Returns y, or (y, x_lam bf16 [M,K]) with keep_x_lam."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    lam = _check_lambda(lam)
    _expect(W_lam, "W_lam", torch.bfloat16)
    if W_lam.dim() != 2 or W_lam.shape[1] != K:
        raise ValueError(f"W_lam must be [N, {K}]")
    N = W_lam.shape[0]
    if y is not None:
        _expect_y(y, M, N)
    lib = load_library()
    _need_cuda(x, gamma, W_lam, y)
    dev = x.device
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=dev)
    x_lam = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if keep_x_lam else None
    ws = None
    if x_lam is None:
        nb = int(lib.bitnet_warmup_forward_workspace_bytes(M, N, K))
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    _check("bitnet_warmup_forward", lib.bitnet_warmup_forward(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), _ptr(W_lam), M, N, K,
        ctypes.c_float(lam), _ptr(y), _dtype_code(y.dtype), _ptr(x_lam), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(stream)))
    return (y, x_lam) if keep_x_lam else y


def bitnet_warmup_backward(dy, x_lam, W_lam, need_dx=True, need_dW=True, stream=None):
    """Straight-through backward of y = x_lam W_lam^T: (dx fp32 [M,K] = dy
    W_lam, dW fp32 [N,K] = dy^T x_lam); either may be skipped (None)."""
    _expect(dy, "dy", torch.bfloat16)
    _expect(x_lam, "x_lam", torch.bfloat16)
    _expect(W_lam, "W_lam", torch.bfloat16)
    M, N = dy.shape
    K = x_lam.shape[1]
    if x_lam.shape != (M, K) or W_lam.shape != (N, K):
        raise ValueError("shapes: dy [M,N], x_lam [M,K], W_lam [N,K]")
    lib = load_library()
    _need_cuda(dy, x_lam, W_lam)
    dev = dy.device
    dx = torch.empty((M, K), dtype=torch.float32, device=dev) if need_dx else None
    dW = torch.empty((N, K), dtype=torch.float32, device=dev) if need_dW else None
    nb = int(lib.bitnet_warmup_backward_workspace_bytes(M, N, K))
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    _check("bitnet_warmup_backward", lib.bitnet_warmup_backward(
        _ptr(dy), _ptr(x_lam), _ptr(W_lam), M, N, K, _ptr(dx), _ptr(dW), _ptr(ws), ws.numel(),
        _stream(stream)))
    return dx, dW


def bitnet_bitdelta_compress(W_base, W_fine, signs=None, alpha=None, stream=None):
    """W_base, W_fine bf16 [N,K] -> (signs int32 [N, K/32] (the bit patterns of
    the uint32 words), alpha fp32 [1])."""
    _expect(W_base, "W_base", torch.bfloat16)
    _expect(W_fine, "W_fine", torch.bfloat16)
    if W_base.dim() != 2 or W_fine.shape != W_base.shape:
        raise ValueError("W_base and W_fine must both be [N, K]")
    N, K = W_base.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    if signs is not None:
        _expect(signs, "signs", torch.int32, numel=N * (K // 32))
    if alpha is not None:
        _expect(alpha, "alpha", torch.float32, numel=1)
    lib = load_library()
    _need_cuda(W_base, W_fine, signs, alpha)
    dev = W_base.device
    if signs is None:
        signs = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
    if alpha is None:
        alpha = torch.empty((1,), dtype=torch.float32, device=dev)
    nb = int(lib.bitnet_bitdelta_compress_workspace_bytes(N, K))
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    _check("bitnet_bitdelta_compress", lib.bitnet_bitdelta_compress(
        _ptr(W_base), _ptr(W_fine), N, K, _ptr(signs), _ptr(alpha), _ptr(ws), ws.numel(),
        _stream(stream)))
    return signs, alpha


def bitnet_bitdelta_forward(x, W_base, signs, alpha, y_dtype=torch.float32, y=None, stream=None):
    """B <= 8 tenants, one token each: x bf16 [B,K], W_base bf16 [N,K], signs
    int32 [B, N, K/32], alpha fp32 [B] -> y [B,N] = x W_base^T + alpha_b x Sign_b^T."""
    _expect(x, "x", torch.bfloat16)
    _expect(W_base, "W_base", torch.bfloat16)
    _expect(signs, "signs", torch.int32)
    _expect(alpha, "alpha", torch.float32)
    B, K = x.shape
    N = W_base.shape[0]
    if W_base.shape != (N, K) or signs.numel() != B * N * (K // 32) or alpha.numel() != B:
        raise ValueError("shapes: x [B,K], W_base [N,K], signs [B,N,K/32], alpha [B]")
    if y is not None:
        _expect_y(y, B, N)
    lib = load_library()
    _need_cuda(x, W_base, signs, alpha, y)
    if y is None:
        y = torch.empty((B, N), dtype=y_dtype, device=x.device)
    _check("bitnet_bitdelta_forward", lib.bitnet_bitdelta_forward(
        _ptr(x), _ptr(W_base), _ptr(signs), _ptr(alpha), B, N, K, _ptr(y),
        _dtype_code(y.dtype), _stream(stream)))
    return y


def _weights_ptr_layout(W, K):
    """(pointer, layout code, N) of row-major packed weights or TiledWeights."""
    if isinstance(W, TiledWeights):
        if W.K != K:
            raise ValueError(f"tiled weights hold K={W.K}, the input has K={K}")
        _need_cuda(W.data)
        return W.data.data_ptr(), BITNET_LAYOUT_TILED, W.N
    N = _expect_packed(W, K)
    _need_cuda(W)
    return W.data_ptr(), BITNET_LAYOUT_ROWS, N


def grouped_problems(items):
    """items: iterable of (x, gamma, eps, W, s_w, y), W row-major packed
    weights [N, K/4] or TiledWeights -> ctypes array of LinearProblem (keep
    the tensors alive while it is used)."""
    items = list(items)
    arr = (LinearProblem * max(1, len(items)))()
    for i, (x, gamma, eps, W, s_w, y) in enumerate(items):
        M, K = _expect_x(x)
        _expect_gamma(gamma, K)
        if not isinstance(W, TiledWeights):
            _expect_packed(W, K)
        _expect_scale(s_w)
        _expect_y(y, M, W.shape[0])
        _need_cuda(x, gamma, s_w, y)
        wp, layout, N = _weights_ptr_layout(W, K)
        arr[i] = LinearProblem(x.data_ptr(), _dtype_code(x.dtype),
                               None if gamma is None else gamma.data_ptr(), float(eps),
                               wp, s_w.data_ptr(), M, N, K,
                               y.data_ptr(), _dtype_code(y.dtype), layout)
    return arr, len(items)


def bitnet_linear_forward_ex(x, gamma, eps, W, s_w, y_dtype=torch.float32, y=None,
                             path=BITNET_PATH_AUTO, want_y=True, debug=True, workspace=None,
                             stream=None):
    """One forward on row-major or tiled weights (W: uint8 [N, K/4] or
    TiledWeights).  With debug, also returns x_q (natural order), s_x and the
    int32 accumulators."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    if not isinstance(W, TiledWeights):
        _expect_packed(W, K)
    N = W.shape[0]
    _expect_scale(s_w)
    _dtype_code(y_dtype)
    if y is not None:
        _expect_y(y, M, N)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8,
                numel=bitnet_linear_forward_workspace_bytes(M, N, K))
    _need_cuda(x, gamma, s_w, y, workspace)
    wp, layout, _ = _weights_ptr_layout(W, K)
    dev = x.device
    if y is None and want_y:
        y = torch.empty((M, N), dtype=y_dtype, device=dev)
    x_q = torch.empty((M, K), dtype=torch.int8, device=dev) if debug else None
    s_x = torch.empty((M,), dtype=torch.float32, device=dev) if debug else None
    acc = torch.empty((M, N), dtype=torch.int32, device=dev) if debug else None
    ws = _ws_for(M, N, K, dev, workspace, stream)
    prob = LinearProblem(x.data_ptr(), _dtype_code(x.dtype),
                         None if gamma is None else gamma.data_ptr(), float(eps), wp,
                         s_w.data_ptr(), M, N, K, None if y is None else y.data_ptr(),
                         _dtype_code(y.dtype if y is not None else y_dtype), layout)
    _check("bitnet_linear_forward_ex", load_library().bitnet_linear_forward_ex(
        ctypes.byref(prob), _ptr(ws), ws.numel(), _ptr(x_q), _ptr(s_x), _ptr(acc), int(path),
        _stream(stream)))
    return {"y": y, "x_q": x_q, "s_x": s_x, "acc": acc}


def bitnet_linear_forward_grouped_workspace_bytes(problems, count):
    return int(load_library().bitnet_linear_forward_grouped_workspace_bytes(
        count, ctypes.cast(problems, ctypes.c_void_p)))


def bitnet_linear_forward_grouped(items, workspace=None, phases=BITNET_PHASE_ALL, stream=None):
    """Run several independent forwards in one call.  items: list of
    (x, gamma, eps, W_packed, s_w, y) with y preallocated [M, N]."""
    items = list(items)
    arr, count = grouped_problems(items)
    nb = bitnet_linear_forward_grouped_workspace_bytes(arr, count)
    if workspace is None:
        workspace = _default_ws.get(nb, items[0][0].device if items else 0, stream)
    _expect(workspace, "workspace", torch.uint8, numel=nb)
    _need_cuda(workspace)
    _check("bitnet_linear_forward_grouped", load_library().bitnet_linear_forward_grouped(
        count, ctypes.cast(arr, ctypes.c_void_p), _ptr(workspace), workspace.numel(),
        int(phases), _stream(stream)))
    return [it[5] for it in items]


def bitnet_linear_forward_debug(x, gamma, eps, W_packed, s_w, y_dtype=torch.float32,
                                path=BITNET_PATH_AUTO, want_y=True, workspace=None,
                                stream=None):
    """Forward that also returns x_q (natural order), s_x and the int32 accumulators."""
    M, K = _expect_x(x)
    _expect_gamma(gamma, K)
    N = _expect_packed(W_packed, K)
    _expect_scale(s_w)
    _dtype_code(y_dtype)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8,
                numel=bitnet_linear_forward_workspace_bytes(M, N, K))
    _need_cuda(x, gamma, W_packed, s_w, workspace)
    dev = x.device
    y = torch.empty((M, N), dtype=y_dtype, device=dev) if want_y else None
    x_q = torch.empty((M, K), dtype=torch.int8, device=dev)
    s_x = torch.empty((M,), dtype=torch.float32, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev)
    ws = _ws_for(M, N, K, dev, workspace, stream)
    _check("bitnet_linear_forward_debug", load_library().bitnet_linear_forward_debug(
        _ptr(x), _dtype_code(x.dtype), _ptr(gamma), float(eps), _ptr(W_packed), _ptr(s_w),
        M, N, K, _ptr(y), _dtype_code(y_dtype), _ptr(ws), ws.numel(), _ptr(x_q), _ptr(s_x),
        _ptr(acc), int(path), _stream(stream)))
    return {"y": y, "x_q": x_q, "s_x": s_x, "acc": acc}


def bitnet_ternary_matmul_i32(x_q, W_packed, path=BITNET_PATH_AUTO, acc=None, workspace=None,
                              stream=None):
    """acc int32 [M,N] = x_q (int8 [M,K]) times the ternary weights transposed."""
    if x_q.dim() != 2:
        raise ValueError("x_q must be 2-D [M, K]")
    _expect(x_q, "x_q", torch.int8)
    M, K = x_q.shape
    N = _expect_packed(W_packed, K)
    if acc is not None:
        _expect(acc, "acc", torch.int32, numel=M * N)
    if workspace is not None:
        _expect(workspace, "workspace", torch.uint8,
                numel=bitnet_linear_forward_workspace_bytes(M, N, K))
    _need_cuda(x_q, W_packed, acc, workspace)
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=x_q.device)
    ws = _ws_for(M, N, K, x_q.device, workspace, stream)
    _check("bitnet_ternary_matmul_i32", load_library().bitnet_ternary_matmul_i32(
        _ptr(x_q), _ptr(W_packed), M, N, K, _ptr(acc), _ptr(ws), ws.numel(), int(path),
        _stream(stream)))
    return acc


def bitnet_device_status(reset=True, stream=None):
    """(status, detail) of the device status word; synchronises the stream."""
    detail = ctypes.c_int(0)
    code = load_library().bitnet_device_status(_stream(stream), 1 if reset else 0,
                                               ctypes.byref(detail))
    return int(code), int(detail.value)


def bitnet_selftest_bounded_wait(limit_ns: int, stream=None):
    _check("bitnet_selftest_bounded_wait",
           load_library().bitnet_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def bitnet_selftest_mma_i8(iters, ctas, a_in_tmem=False, stream=None):
    """Queue the int8 tensor-core rate kernel (see the header); returns the
    int8 operation count it performs."""
    _check("bitnet_selftest_mma_i8", load_library().bitnet_selftest_mma_i8(
        int(iters), int(ctas), 1 if a_in_tmem else 0, _stream(stream)))
    return 2 * 128 * 256 * 32 * int(iters) * int(ctas)


def bitnet_selftest_divide(a, b, stream=None):
    """a / b (fp32 CUDA tensors) through the decode epilogue's division."""
    _expect(a, "a", torch.float32)
    _expect(b, "b", torch.float32, numel=a.numel())
    _need_cuda(a, b)
    a = a.contiguous()
    b = b.contiguous()
    q = torch.empty_like(a)
    _check("bitnet_selftest_divide",
           load_library().bitnet_selftest_divide(_ptr(a), _ptr(b), _ptr(q), a.numel(),
                                                 _stream(stream)))
    return q


class BitLinear:
    """A linear layer y = x W^T with ternary weights, packed once on creation.

    Holds W_packed (uint8 [N, K/4]), s_w (fp32 [1]) and the RMSNorm gain."""

    def __init__(self, W, gamma=None, eps=1e-5):
        self.W_packed, self.s_w = bitnet_quantize_pack_weights(W.contiguous())
        self.gamma = gamma
        self.eps = float(eps)
        self.out_features, self.in_features = W.shape

    def __call__(self, x, y_dtype=torch.bfloat16, y=None, stream=None):
        return bitnet_linear_forward(x, self.gamma, self.eps, self.W_packed, self.s_w,
                                     y_dtype=y_dtype, y=y, stream=stream)
