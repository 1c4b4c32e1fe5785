"""The allocation-free weight quantization entry point.

bitnet_quantize_pack_weights_static exists for callers that cannot allocate
device memory (for example a plugin whose host engine owns the whole memory
budget and passes it only its tensors, or code that must not risk the
device-wide synchronisation of cudaMalloc/cudaFree).  It keeps its scratch in
a static device array inside the library.  This test calls it through the C
ABI twice in a row and checks both results against the regular
(workspace-taking) entry point, bit for bit like every other packed-weight
comparison in the suite.  The file runs last so that a failure here cannot
hide failures elsewhere, and it sets up everything it needs so it also passes
alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_quantized_linear_b200 as tql
from ternary_quantized_linear_b200 import build as tql_build
from ternary_quantized_linear_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    tql_build.build()
    torch.cuda.set_device(0)
    return tql.load_library()


def _static_call(lib, W):
    N, K = W.shape
    W_p = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    s_w = torch.empty((1,), dtype=torch.float32, device=W.device)
    rc = lib.bitnet_quantize_pack_weights_static(
        ctypes.c_void_p(W.data_ptr()), N, K, ctypes.c_void_p(W_p.data_ptr()),
        ctypes.c_void_p(s_w.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == tql.BITNET_OK, tql.bitnet_status_string(rc)
    return W_p, s_w


def test_static_scratch_matches_workspace_entry_on_two_calls(lib):
    mats = [workloads.weights(workloads.CASES[1], 1),   # 8640 x 3200
            workloads.weights(workloads.CASES[0], 0)]   # 512 x 256
    for W_np in mats:
        W = torch.from_numpy(W_np).cuda()
        got_p, got_s = _static_call(lib, W)
        ref_p, ref_s = tql.bitnet_quantize_pack_weights(W)
        torch.cuda.synchronize()
        assert np.array_equal(got_p.cpu().numpy(), ref_p.cpu().numpy())
        assert got_s.cpu().numpy().tobytes() == ref_s.cpu().numpy().tobytes()


def test_static_scratch_rejects_rows_beyond_its_limit(lib):
    N, K = tql.BITNET_STATIC_SCRATCH_MAX_N + 1, 64
    W = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    W_p = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    s_w = torch.empty((1,), dtype=torch.float32, device="cuda")
    rc = lib.bitnet_quantize_pack_weights_static(
        ctypes.c_void_p(W.data_ptr()), N, K, ctypes.c_void_p(W_p.data_ptr()),
        ctypes.c_void_p(s_w.data_ptr()), None)
    assert rc == tql.BITNET_ERR_SCRATCH_LIMIT
    assert "65536" in tql.bitnet_status_string(rc)
