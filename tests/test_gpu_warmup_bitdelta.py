"""Parity of the quantization warm-up (forward and straight-through
backward) and of BitDelta (compression and the multi-tenant forward) with
the oracle.

Warm-up ("LLM を 1.58 ビットにファインチューニング", 動的ウォームアップ量子化):
the bf16 operands W_lam and x_lam are compared bit for bit with the oracle's
fp32 operands rounded to bf16; y, dx and dW, sums of bf16 products on the
tensor cores, within the fp32 accumulation bound derived below.
BitDelta (Eq. 1-4, 6): sign words and alpha bit for bit; y within the same
bound.

Accumulation bound: the products of bf16 operands are exact in fp32, so the
only error of a length-K dot product is the fp32 summation.  The tensor
cores add K/16 partial sums of 16 products into an fp32 accumulator; with
unit roundoff u = 2^-24 per addition and at most 2 u for each internal
16-term sum, |y - y_exact| <= (K/16 + 32) * 2 u * sum|products|.  The test
allows (K/16 + 64) * 2^-23 * sum|products| (plus half a bf16 ulp of y for
bf16 outputs).
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_quantized_linear_b200 as tql
from ternary_quantized_linear_b200 import workloads

from _util import bf16_bits, sample_columns, x_to_device

pytestmark = pytest.mark.gpu


def _bound(K, absdot):
    return (K / 16 + 64) * 2.0 ** -23 * absdot


def _bits_to_dev(b):
    return x_to_device(np.ascontiguousarray(b, np.uint16))


# ----------------------------------------------------------------- warm-up

@pytest.mark.parametrize("lam", [0.0, 0.3, 1.0])
@pytest.mark.parametrize("N,K", [(64, 256), (208, 768), (1024, 4096)])
def test_warmup_weight_operand_bits(N, K, lam):
    W, _, _ = workloads.warmup_inputs(1, N, K, seed=1)
    W_lam, s_w = tql.bitnet_warmup_quantize_weights(torch.from_numpy(W).cuda(), lam)
    torch.cuda.synchronize()
    ref, ref_s = oracle.warmup_weights(W, lam)
    assert np.float32(s_w.item()) == ref_s
    assert np.array_equal(bf16_bits(W_lam), oracle.f32_to_bf16(ref))


@pytest.mark.parametrize("x_f32", [False, True])
@pytest.mark.parametrize("lam", [0.0, 0.45, 1.0])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (5, 208, 768), (64, 1024, 4096),
                                   (300, 520, 1024)])
def test_warmup_forward_matches_oracle(M, N, K, lam, x_f32):
    W, x, _ = workloads.warmup_inputs(M, N, K, seed=2, f32=x_f32)
    gamma = workloads.random_gamma(K)
    W_lam, _ = tql.bitnet_warmup_quantize_weights(torch.from_numpy(W).cuda(), lam)
    xd = x_to_device(x)
    gd = torch.from_numpy(gamma).cuda()
    y, x_lam = tql.bitnet_warmup_forward(xd, gd, 1e-5, W_lam, lam, keep_x_lam=True)
    torch.cuda.synchronize()
    ref = oracle.warmup_forward(x, gamma, 1e-5, W, lam)
    assert np.array_equal(bf16_bits(x_lam), oracle.f32_to_bf16(ref["x_lam"]))
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref["y_b"])
    assert np.all(err <= _bound(K, ref["absdot"]))


def test_warmup_forward_large_sampled_bf16_output():
    M, N, K = 2048, 4096, 4096
    W, x, _ = workloads.warmup_inputs(M, N, K, seed=3)
    W_lam, _ = tql.bitnet_warmup_quantize_weights(torch.from_numpy(W).cuda(), 0.6)
    y = tql.bitnet_warmup_forward(x_to_device(x), None, 1e-5, W_lam, 0.6, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    cols = sample_columns(N, 96, seed=5)
    rows = np.array(sorted({0, 1, 127, 128, 255, 256, 1000, M - 1}), np.int64)
    ref = oracle.warmup_forward(x[rows], None, 1e-5, W, 0.6, cols)
    got = bf16_bits(y)[rows][:, cols]
    got = oracle.bf16_bits_to_f32(got).astype(np.float64)
    err = np.abs(got - ref["y_b"])
    assert np.all(err <= _bound(K, ref["absdot"]) + 2.0 ** -8 * np.abs(ref["y_b"]))


@pytest.mark.parametrize("M,N,K", [(1, 64, 256), (7, 208, 512), (130, 256, 1024),
                                   (512, 1024, 2048)])
def test_warmup_backward_matches_oracle(M, N, K):
    W, x, dy = workloads.warmup_inputs(M, N, K, seed=4)
    W_lam, _ = tql.bitnet_warmup_quantize_weights(torch.from_numpy(W).cuda(), 0.7)
    _, x_lam = tql.bitnet_warmup_forward(x_to_device(x), None, 1e-5, W_lam, 0.7, keep_x_lam=True)
    dyd = _bits_to_dev(dy)
    dx, dW = tql.bitnet_warmup_backward(dyd, x_lam, W_lam)
    torch.cuda.synchronize()
    xl_b, wl_b = bf16_bits(x_lam), bf16_bits(W_lam)
    rdx, rdW = oracle.warmup_backward(dy, xl_b, wl_b)
    a_dy = np.abs(oracle.bf16_bits_to_f32(dy).astype(np.float64))
    a_x = np.abs(oracle.bf16_bits_to_f32(xl_b).astype(np.float64))
    a_w = np.abs(oracle.bf16_bits_to_f32(wl_b).astype(np.float64))
    assert np.all(np.abs(dx.cpu().numpy() - rdx) <= _bound(N, a_dy @ a_w))
    assert np.all(np.abs(dW.cpu().numpy() - rdW) <= _bound(M, a_dy.T @ a_x))
    dx2, dW2 = tql.bitnet_warmup_backward(dyd, x_lam, W_lam, need_dx=False)
    torch.cuda.synchronize()
    assert dx2 is None and torch.equal(dW2, dW)


def test_warmup_rejects_bad_lambda_and_shapes():
    W = torch.zeros((64, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        tql.bitnet_warmup_quantize_weights(W, 1.5)
    with pytest.raises(tql.BitnetError):
        tql.bitnet_warmup_quantize_weights(torch.zeros((63, 256), device="cuda"), 0.5)


# ---------------------------------------------------------------- BitDelta

@pytest.mark.parametrize("N,K", [(64, 256), (300, 1024), (1024, 4096)])
def test_bitdelta_compress_matches_oracle(N, K):
    base, fine, _ = workloads.bitdelta_inputs(N, K, 2, seed=1)
    bd = _bits_to_dev(base)
    for f in fine:
        signs, alpha = tql.bitnet_bitdelta_compress(bd, _bits_to_dev(f))
        torch.cuda.synchronize()
        rs, ra, _ = oracle.bitdelta_compress(base, f)
        assert np.array_equal(signs.cpu().numpy().view(np.uint32), rs)
        assert np.float32(alpha.item()) == ra


def _bitdelta_case(N, K, B, seed, cols=None, y_dtype=torch.float32):
    base, fine, x = workloads.bitdelta_inputs(N, K, B, seed=seed)
    bd = _bits_to_dev(base)
    signs = torch.empty((B, N, K // 32), dtype=torch.int32, device="cuda")
    alpha = torch.empty((B,), dtype=torch.float32, device="cuda")
    for b in range(B):
        tql.bitnet_bitdelta_compress(bd, _bits_to_dev(fine[b]), signs=signs[b], alpha=alpha[b:b + 1])
    y = tql.bitnet_bitdelta_forward(_bits_to_dev(x), bd, signs, alpha, y_dtype=y_dtype)
    torch.cuda.synchronize()
    s_np = signs.cpu().numpy().view(np.uint32)
    ref, absdot = oracle.bitdelta_forward(x, base, s_np, alpha.cpu().numpy(), cols)
    if y_dtype == torch.float32:
        got = y.cpu().numpy().astype(np.float64)
    else:
        got = oracle.bf16_bits_to_f32(bf16_bits(y)).astype(np.float64)
    if cols is not None:
        got = got[:, cols]
    err = np.abs(got - ref)
    tol = _bound(K, absdot)
    if y_dtype != torch.float32:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    assert np.all(err <= tol)


@pytest.mark.parametrize("B", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(64, 256), (200, 1024), (1000, 2048)])
def test_bitdelta_forward_matches_oracle(N, K, B):
    _bitdelta_case(N, K, B, seed=2)


def test_bitdelta_forward_fig4_shape_sampled():
    """The page's Fig. 4 setting: an 8192 x 8192 layer, 8 tenants."""
    N = K = 8192
    _bitdelta_case(N, K, 8, seed=3, cols=sample_columns(N, 128, seed=1))


def test_bitdelta_forward_bf16_output():
    _bitdelta_case(520, 1024, 5, seed=4, y_dtype=torch.bfloat16)


def test_warmup_and_bitdelta_leave_no_device_failure():
    code, _ = tql.bitnet_device_status(reset=False)
    assert code == 0


def test_bitdelta_forward_odd_word_count_and_unaligned_signs():
    """K/32 not a multiple of 4 and a sign buffer that is only 4-byte
    aligned: the kernel falls back from its 16-byte sign loads."""
    N, K, B = 96, 1056, 3
    base, fine, x = workloads.bitdelta_inputs(N, K, B, seed=6)
    bd = _bits_to_dev(base)
    buf = torch.empty(B * N * (K // 32) + 1, dtype=torch.int32, device="cuda")
    signs = buf[1:].view(B, N, K // 32)
    alpha = torch.empty((B,), dtype=torch.float32, device="cuda")
    for b in range(B):
        tql.bitnet_bitdelta_compress(bd, _bits_to_dev(fine[b]), signs=signs[b], alpha=alpha[b:b + 1])
    y = tql.bitnet_bitdelta_forward(_bits_to_dev(x), bd, signs, alpha)
    torch.cuda.synchronize()
    ref, absdot = oracle.bitdelta_forward(x, base, signs.cpu().numpy().view(np.uint32),
                                          alpha.cpu().numpy())
    assert np.all(np.abs(y.cpu().numpy() - ref) <= _bound(K, absdot))
