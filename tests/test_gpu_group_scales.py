"""Parity of the group-wise-scale forward with the oracle.

Group-wise scales (bitnet.cpp article, グループ量子化と正規化, applied to the
absmean / absmax scheme of the BitNet fine-tuning article, 量子化の仕組み):
the weights and activations are split into K/group_k groups along K, each
with its own scale.  The weight scales and packed codes, the activation codes
and scales, the per-group int32 sums and y (fp64 sum of the fp32 group terms,
rounded once) are all compared bit for bit with the oracle, on both matmul
paths (the tiled decode kernel for M <= 16 on tiled weights, the tcgen05
kernel otherwise).
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_quantized_linear_b200 as tql
from ternary_quantized_linear_b200 import workloads

from _util import bf16_bits, sample_columns, x_to_device

pytestmark = pytest.mark.gpu


def _weights(N, K, gk, seed=0):
    W = workloads.group_scaled_weights(N, K, gk, seed)
    Wd = torch.from_numpy(W).cuda()
    W_p, s_w = tql.bitnet_quantize_pack_weights_group_scales(Wd, gk)
    torch.cuda.synchronize()
    ref_s = oracle.group_weight_scale(W, gk)
    ref_p = oracle.group_quantize_pack(W, gk, ref_s)
    return W, W_p, s_w, ref_p, ref_s


@pytest.mark.parametrize("N,K,gk", [(96, 1024, 256), (300, 2048, 512), (1024, 4096, 1024),
                                    (129, 768, 256)])
def test_group_weight_scales_and_codes_match_oracle(N, K, gk):
    _, W_p, s_w, ref_p, ref_s = _weights(N, K, gk)
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(W_p.cpu().numpy(), ref_p)


def _check_forward(M, N, K, gk, layout, cols=None, seed=0):
    W, W_p, s_w, ref_p, ref_s = _weights(N, K, gk, seed)
    x = workloads.group_scaled_activations(M, K, gk, seed)
    xd = x_to_device(x)
    Wuse = tql.bitnet_tile_weights(W_p) if layout == "tiled" else W_p
    ref = oracle.group_linear_forward(x, None, workloads.DEFAULT_EPS, ref_p, ref_s, K, gk, cols)
    for ydt in (torch.float32, torch.bfloat16):
        out = tql.bitnet_linear_forward_group_scales(xd, None, workloads.DEFAULT_EPS, Wuse, s_w,
                                                     gk, y_dtype=ydt, debug=True)
        torch.cuda.synchronize()
        assert np.array_equal(out["x_q"].cpu().numpy(), ref["x_q"])
        assert np.array_equal(out["s_x"].cpu().numpy().view(np.uint32), ref["s_x"].view(np.uint32))
        acc = out["acc"].cpu().numpy()                     # [G, M, N]
        if cols is not None:
            acc = acc[:, :, cols]
        assert np.array_equal(acc.transpose(1, 2, 0), ref["acc"])
        y = out["y"]
        if cols is not None:
            y = y[:, torch.from_numpy(cols).cuda()]
        if ydt == torch.float32:
            assert np.array_equal(y.cpu().numpy().view(np.uint32), ref["y"].view(np.uint32))
        else:
            assert np.array_equal(bf16_bits(y), ref["y_bf16"])


@pytest.mark.parametrize("layout", ["rows", "tiled"])
@pytest.mark.parametrize("M", [1, 3, 8, 16, 40, 300])
def test_group_forward_small_shapes_match_oracle(M, layout):
    _check_forward(M, 384, 2048, 512, layout)


@pytest.mark.parametrize("layout", ["rows", "tiled"])
@pytest.mark.parametrize("M,N,K,gk", [(1, 4096, 4096, 1024), (16, 4096, 14336, 2048),
                                      (9, 14336, 4096, 256), (64, 4096, 4096, 4096)])
def test_group_forward_model_shapes_sampled(M, N, K, gk, layout):
    _check_forward(M, N, K, gk, layout, cols=sample_columns(N, 256, seed=M))


@pytest.mark.parametrize("layout", ["rows", "tiled"])
def test_group_forward_ragged(layout):
    _check_forward(5, 200, 768, 256, layout)


@pytest.mark.parametrize("M", [1, 16, 64])
def test_one_group_equals_per_tensor_forward(M):
    """group_k = K: one scale for the tensor, so the group forward must give
    the per-tensor forward's bits exactly."""
    N, K = 640, 2048
    W = workloads.group_scaled_weights(N, K, K, 3)
    Wd = torch.from_numpy(W).cuda()
    W_pg, s_wg = tql.bitnet_quantize_pack_weights_group_scales(Wd, K)
    W_p, s_w = tql.bitnet_quantize_pack_weights(Wd)
    torch.cuda.synchronize()
    assert torch.equal(W_pg, W_p)
    assert torch.equal(s_wg.view(torch.int32), s_w.view(torch.int32))
    xd = x_to_device(workloads.group_scaled_activations(M, K, K, 3))
    y_g = tql.bitnet_linear_forward_group_scales(xd, None, 1e-5, W_p, s_w, K)["y"]
    y = tql.bitnet_linear_forward(xd, None, 1e-5, W_p, s_w, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y_g.view(torch.int32), y.view(torch.int32))


def test_group_scales_leave_no_device_failure():
    code, _ = tql.bitnet_device_status(reset=False)
    assert code == 0
