"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/bitnet_b200.h declares, sizes its workspaces, and
rejects bad arguments before touching the device (the invalid calls below use
fake pointer values that are never dereferenced)."""
import ctypes
import os
import re
import subprocess

import pytest

import ternary_quantized_linear_b200 as tql
from ternary_quantized_linear_b200 import build as tql_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet_b200.h")


@pytest.fixture(scope="module")
def lib():
    tql_build.build()
    return tql.load_library()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"BITNET_API[^;{]*?\b(bitnet_\w+)\s*\(", src, re.S)))


def test_header_declares_the_three_core_calls():
    names = _declared()
    for n in ("bitnet_quantize_pack_weights", "bitnet_rmsnorm_quant_act",
              "bitnet_linear_forward", "bitnet_linear_forward_debug",
              "bitnet_ternary_matmul_i32"):
        assert n in names


def test_binding_limits_mirror_the_header():
    text = open(HEADER).read()
    for name in ("BITNET_MAX_K", "BITNET_MAX_M", "BITNET_MAX_N"):
        expr = re.search(rf"#define {name} (\(.*\))", text).group(1)
        assert eval(expr) == getattr(tql, name), name  # arithmetic on integer literals


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", tql.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(bitnet_\w+)$", out, re.M))
    declared = set(_declared())
    assert declared <= exported, declared - exported
    assert declared == set(tql.EXPORTED)
    # nothing else leaks out of the library
    assert exported == declared


def test_status_strings(lib):
    for code in range(0, 8):
        assert tql.bitnet_status_string(code)
    assert tql.bitnet_status_string(99) == "unknown status"
    assert tql.bitnet_version() >= 100


def test_workspace_sizes(lib):
    assert tql.bitnet_quantize_pack_weights_workspace_bytes(1000, 4096) >= 8000
    small = tql.bitnet_linear_forward_workspace_bytes(16, 3200, 3200)
    # x_q + scales + row sums + split-K int32 partials + counters
    assert small >= 16 * 3200 + 16 * 3200 * 4
    assert small % 256 == 0
    big = tql.bitnet_linear_forward_workspace_bytes(2048, 14336, 4096)
    assert big >= 2048 * 4096 and big < 2048 * 4096 + 64 * 1024
    assert tql.bitnet_linear_forward_workspace_bytes(-1, 1, 64) == 0


FAKE = 0x10000  # 64 KiB-aligned fake device address, never dereferenced


def _fwd(lib, x=FAKE, xd=1, gamma=None, eps=1e-5, wp=FAKE, sw=FAKE, M=4, N=64, K=256,
         y=FAKE, yd=1, ws=FAKE, wsb=1 << 30):
    P = ctypes.c_void_p
    return lib.bitnet_linear_forward(P(x), xd, P(gamma) if gamma else None, ctypes.c_float(eps),
                                     P(wp), P(sw), M, N, K, P(y), yd, P(ws), wsb, None)


def test_forward_rejects_bad_arguments(lib):
    assert _fwd(lib, K=100) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, K=0) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, K=32) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, N=0) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    # the tensor-core grid holds at most 65535 token tiles of 128
    assert _fwd(lib, M=tql.BITNET_MAX_M + 1) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, N=tql.BITNET_MAX_N + 1) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, K=tql.BITNET_MAX_K + 64) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert _fwd(lib, M=-1) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, x=0) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, y=0) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, xd=7) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, eps=-1.0) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, eps=float("nan")) == tql.BITNET_ERR_INVALID_ARG
    assert _fwd(lib, x=FAKE + 8) == tql.BITNET_ERR_MISALIGNED
    assert _fwd(lib, wp=FAKE + 4) == tql.BITNET_ERR_MISALIGNED
    assert _fwd(lib, ws=FAKE + 128) == tql.BITNET_ERR_MISALIGNED
    assert _fwd(lib, wsb=16) == tql.BITNET_ERR_WORKSPACE
    assert _fwd(lib, ws=0) == tql.BITNET_ERR_WORKSPACE
    # empty batch: valid, queues nothing, touches no pointer
    assert _fwd(lib, M=0) == tql.BITNET_OK


def test_other_entry_points_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    assert lib.bitnet_quantize_pack_weights(P(FAKE), 64, 100, P(FAKE), P(FAKE), P(FAKE), 1 << 20,
                                            None) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert lib.bitnet_quantize_pack_weights(P(FAKE), 64, 128, P(FAKE), P(FAKE), P(FAKE), 8,
                                            None) == tql.BITNET_ERR_WORKSPACE
    assert lib.bitnet_quantize_pack_weights(P(FAKE + 4), 64, 128, P(FAKE), P(FAKE), P(FAKE),
                                            1 << 20, None) == tql.BITNET_ERR_MISALIGNED
    assert lib.bitnet_rmsnorm_quant_act(P(FAKE), 0, None, ctypes.c_float(1e-5), 2, 96, P(FAKE),
                                        P(FAKE), None) == tql.BITNET_ERR_UNSUPPORTED_SHAPE
    assert lib.bitnet_rmsnorm_quant_act(P(FAKE), 0, None, ctypes.c_float(1e-5), 0, 128, P(FAKE),
                                        P(FAKE), None) == tql.BITNET_OK
    # the GEMV path is only for M <= 16
    assert lib.bitnet_ternary_matmul_i32(P(FAKE), P(FAKE), 17, 64, 128, P(FAKE), P(FAKE), 1 << 30,
                                         tql.BITNET_PATH_GEMV, None) == tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_ternary_matmul_i32(P(FAKE), P(FAKE), 4, 64, 128, P(FAKE), P(FAKE), 1 << 30,
                                         9, None) == tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_selftest_bounded_wait(10, None) == tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_selftest_divide(P(FAKE), P(FAKE), P(FAKE), -1, None) == \
        tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_selftest_divide(None, P(FAKE), P(FAKE), 4, None) == tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_selftest_divide(P(FAKE + 4), P(FAKE), P(FAKE), 4, None) == \
        tql.BITNET_ERR_MISALIGNED
    assert lib.bitnet_selftest_divide(None, None, None, 0, None) == tql.BITNET_OK


def test_binding_refuses_cpu_tensors(lib):
    import torch
    W = torch.zeros(64, 128)
    with pytest.raises(ValueError):
        tql.bitnet_quantize_pack_weights(W)


def test_grouped_validation_and_workspace(lib):
    import ctypes as C
    P = tql.LinearProblem
    arr = (P * 17)()
    for i in range(17):
        arr[i] = P(FAKE, 1, None, 1e-5, FAKE, FAKE, 4, 64, 256, FAKE, 1)
    ptr = C.cast(arr, C.c_void_p)
    assert lib.bitnet_linear_forward_grouped(17, ptr, C.c_void_p(FAKE), 1 << 30, 3, None) == \
        tql.BITNET_ERR_INVALID_ARG
    assert lib.bitnet_linear_forward_grouped(2, ptr, C.c_void_p(FAKE), 1 << 30, 0, None) == \
        tql.BITNET_ERR_INVALID_ARG
    arr[1].K = 100
    assert lib.bitnet_linear_forward_grouped(2, ptr, C.c_void_p(FAKE), 1 << 30, 3, None) == \
        tql.BITNET_ERR_UNSUPPORTED_SHAPE
    arr[1].K = 256
    arr[1].y = FAKE + 4
    assert lib.bitnet_linear_forward_grouped(2, ptr, C.c_void_p(FAKE), 1 << 30, 3, None) == \
        tql.BITNET_ERR_MISALIGNED
    arr[1].y = FAKE
    one = tql.bitnet_linear_forward_workspace_bytes(4, 64, 256)
    assert tql.bitnet_linear_forward_grouped_workspace_bytes(arr, 2) == 2 * one
    assert lib.bitnet_linear_forward_grouped(2, ptr, C.c_void_p(FAKE), 2 * one - 1, 3, None) == \
        tql.BITNET_ERR_WORKSPACE
    # empty groups and empty problems queue nothing
    assert lib.bitnet_linear_forward_grouped(0, None, None, 0, 3, None) == tql.BITNET_OK
    arr[0].M = 0
    arr[1].M = 0
    assert lib.bitnet_linear_forward_grouped(2, ptr, None, 0, 3, None) == tql.BITNET_OK


def test_unsupported_shape_message_names_every_limit(lib):
    msg = tql.bitnet_status_string(tql.BITNET_ERR_UNSUPPORTED_SHAPE)
    for part in ("65535*128", "2^24", "2^20", "K % 64"):
        assert part in msg


def test_spec_named_utilities_agree(lib):
    for M, N, K in ((1, 64, 64), (16, 3200, 8640), (2048, 14336, 4096)):
        assert lib.bitnet_workspace_bytes(M, N, K) == \
            tql.bitnet_linear_forward_workspace_bytes(M, N, K)


def _cpu(shape, dtype):
    import torch
    return torch.zeros(shape, dtype=dtype)


def test_binding_rejects_wrong_buffers_before_the_library(lib):
    # CPU tensors: every check below must fire before the CUDA-tensor check,
    # i.e. before any pointer could reach the library.
    import torch
    M, N, K = 4, 64, 256
    x = _cpu((M, K), torch.bfloat16)
    W_p = _cpu((N, K // 4), torch.uint8)
    s_w = _cpu((1,), torch.float32)
    y = _cpu((M, N), torch.bfloat16)
    cases = [
        (TypeError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p.view(torch.int8), s_w, y=y)),
        (ValueError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, _cpu((N, K // 8), torch.uint8),
                                                       s_w, y=y)),
        (TypeError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w.double(), y=y)),
        (ValueError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p, _cpu((0,), torch.float32),
                                                       y=y)),
        (ValueError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w,
                                                       y=_cpu((M, N - 1), torch.bfloat16))),
        (TypeError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w,
                                                      y=_cpu((M, N), torch.float16))),
        (ValueError, lambda: tql.bitnet_linear_forward(x, _cpu((K - 1,), torch.float32), 1e-5, W_p,
                                                       s_w, y=y)),
        (ValueError, lambda: tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w, y=y,
                                                       workspace=_cpu((16,), torch.uint8))),
        (TypeError, lambda: tql.bitnet_linear_forward(x.half(), None, 1e-5, W_p, s_w, y=y)),
        (ValueError, lambda: tql.bitnet_quantize_pack_weights_static(
            _cpu((N, K), torch.float32), _cpu((N, K // 4 - 1), torch.uint8), s_w)),
        (TypeError, lambda: tql.bitnet_quantize_pack_weights_static(
            _cpu((N, K), torch.float32), W_p, _cpu((1,), torch.float16))),
        (ValueError, lambda: tql.bitnet_quantize_pack_weights(
            _cpu((N, K), torch.float32), W_packed=_cpu((N, K // 4 - 1), torch.uint8))),
        (ValueError, lambda: tql.bitnet_rmsnorm_quant_act(x, None, 1e-5,
                                                          x_q=_cpu((M, K - 1), torch.int8))),
        (ValueError, lambda: tql.bitnet_rmsnorm_quant_act(x, None, 1e-5,
                                                          s_x=_cpu((M - 1,), torch.float32))),
        (TypeError, lambda: tql.bitnet_ternary_matmul_i32(_cpu((M, K), torch.int8), W_p,
                                                          acc=_cpu((M, N), torch.int64))),
        (ValueError, lambda: tql.bitnet_linear_matmul(W_p, s_w, M, K, _cpu((16,), torch.uint8))),
        (ValueError, lambda: tql.grouped_problems([(x, None, 1e-5, W_p, s_w,
                                                    _cpu((M + 1, N), torch.bfloat16))])),
    ]
    for exc, call in cases:
        with pytest.raises(exc):
            call()
