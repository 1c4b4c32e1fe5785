"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a hand-worked example, brute force through a library integer
matmul, exact (correctly rounded) sums, closed-form statistics, fp64
re-derivations within their rounding bounds, and symmetries the method must
have.  A dropped term, a wrong sign or index, a transposed operand or
half-away-from-zero rounding each fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bitlinear_4x4.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _bf16_bits(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------- golden 4x4 case

def test_golden_4x4_weights():
    g = _golden()
    W = np.array(g["W"], np.float32)
    s_w, S = oracle.weight_scale(W)
    assert S == g["sum_abs_W"]
    assert s_w == np.float32(g["s_w"])
    W_p, T = oracle.quantize_pack(W, s_w)
    assert T.tolist() == g["T"]
    assert W_p.ravel().tolist() == g["W_p"]
    assert oracle.unpack(W_p, 4).tolist() == g["T"]


@pytest.mark.parametrize("as_bf16", [False, True])
def test_golden_4x4_forward(as_bf16):
    g = _golden()
    W = np.array(g["W"], np.float32)
    x = np.array(g["x"], np.float32)
    if as_bf16:
        x = _bf16_bits(x)  # every value is exact in bf16
    gamma = np.array(g["gamma"], np.float32)
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    r = oracle.linear_forward(x, gamma, g["eps"], W_p, s_w, 4)
    assert r["s_x"].tolist() == g["s_x"]
    assert r["x_q"].tolist() == g["x_q"]
    assert r["acc"].tolist() == g["acc"]
    assert r["y"].tolist() == g["y"]
    assert r["y_bf16"].tolist() == _bf16_bits(np.array(g["y"], np.float32)).tolist()
    assert r["rowsum"].tolist() == np.array(g["x_q"]).sum(1).tolist()


def test_golden_ties_are_to_even():
    # mean|W| = 0.5 -> s_w = 2; products land exactly on +-0.5 and +-1.5
    W = np.array([[0.25, -0.25, 0.75, -0.75]], np.float32)
    s_w, _ = oracle.weight_scale(W)
    assert s_w == 2.0
    _, T = oracle.quantize_pack(W, s_w)
    assert T.tolist() == [[0, 0, 1, -1]]
    # activations: x_n * s_x = +-62.5 / +-33.5 (see golden) -> 62 / 34


# ------------------------------------------------------------- packing

def test_pack_roundtrip_and_no_code_3():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((37, 128)) * 0.02).astype(np.float32)
    s_w, _ = oracle.weight_scale(W)
    W_p, T = oracle.quantize_pack(W, s_w)
    assert set(np.unique(T).tolist()) <= {-1, 0, 1}
    assert np.array_equal(oracle.unpack(W_p, 128), T)
    fields = np.stack([(W_p >> (2 * j)) & 3 for j in range(4)], -1)
    assert not np.any(fields == 3)
    assert W_p.shape == (37, 32)  # four weights per byte


def test_weight_sign_symmetry():
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    s1, _ = oracle.weight_scale(W)
    s2, _ = oracle.weight_scale(-W)
    assert s1 == s2
    _, T1 = oracle.quantize_pack(W, s1)
    _, T2 = oracle.quantize_pack(-W, s2)
    assert np.array_equal(T1, -T2)


def test_zero_weights():
    W = np.zeros((8, 64), np.float32)
    s_w, S = oracle.weight_scale(W)
    assert S == 0.0
    assert s_w == np.float32(1.0) / np.float32(1e-5)
    W_p, T = oracle.quantize_pack(W, s_w)
    assert not T.any()
    assert np.all(W_p == 0x55)


# ------------------------------------------------------------- weight scale

@pytest.mark.parametrize("shape", [(3, 64), (257, 1024), (600, 4096)])
def test_weight_scale_matches_exact_sum(shape):
    rng = np.random.default_rng(3)
    W = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    s_w, S = oracle.weight_scale(W)
    exact = math.fsum(np.abs(W.astype(np.float64)).ravel().tolist())
    assert abs(S - exact) <= 1e-13 * exact
    mean32 = np.float32(exact / (shape[0] * shape[1]))
    want = np.float32(1.0) / mean32
    assert abs(float(s_w) - float(want)) <= float(np.spacing(want))


@pytest.mark.parametrize("sigma", [0.02, 0.015])
def test_weight_scale_statistics(sigma):
    # W ~ N(0, sigma^2): E|W| = sigma sqrt(2/pi); a weight is 0 when
    # |w| s_w <= 1/2, i.e. |w| <= E|W|/2, probability 2 Phi(sqrt(2/pi)/2) - 1
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((1024, 2048)) * sigma).astype(np.float32)
    s_w, _ = oracle.weight_scale(W)
    expect = 1.0 / (sigma * math.sqrt(2.0 / math.pi))
    assert abs(float(s_w) / expect - 1.0) < 1e-3
    _, T = oracle.quantize_pack(W, s_w)
    zero_frac = float(np.mean(T == 0))
    phi = 0.5 * (1.0 + math.erf(0.5 * math.sqrt(2.0 / math.pi) / math.sqrt(2.0)))
    assert abs(zero_frac - (2.0 * phi - 1.0)) < 0.01
    assert abs(float(np.mean(T == 1)) - float(np.mean(T == -1))) < 0.01


# ---------------------------------------------------------- activations

@pytest.mark.parametrize("K", [64, 256, 3200, 28672])
def test_rmsnorm_matches_fp64(K):
    rng = np.random.default_rng(K)
    x = rng.standard_normal((5, K)).astype(np.float32)
    x[:, :3] *= 20.0
    gamma = workloads.random_gamma(K)
    eps = 1e-5
    _, _, _, xn = oracle.rmsnorm_quant_act(x, gamma, eps)
    x64 = x.astype(np.float64)
    ref = x64 * gamma.astype(np.float64) / np.sqrt((x64 ** 2).mean(1, keepdims=True) + eps)
    rel = np.abs(xn - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() < 2e-5
    assert np.median(rel) < 1e-6


def test_act_quant_matches_fp64_decisions():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 4096)).astype(np.float32)
    x_q, s_x, _, _ = oracle.rmsnorm_quant_act(x, None, 1e-5)
    x64 = x.astype(np.float64)
    xn = x64 / np.sqrt((x64 ** 2).mean(1, keepdims=True) + 1e-5)
    amax = np.abs(xn).max(1, keepdims=True)
    assert np.allclose(s_x, 127.0 / amax[:, 0], rtol=2e-5)
    q = np.clip(np.rint(xn * 127.0 / amax), -128, 127)
    diff = x_q.astype(np.int64) - q.astype(np.int64)
    assert np.abs(diff).max() <= 1
    assert np.count_nonzero(diff) <= 1e-4 * diff.size


def test_act_quant_invariants():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((16, 512)).astype(np.float32)
    x[:, 5] *= 20.0
    x_q, s_x, rs, _ = oracle.rmsnorm_quant_act(x, None, 0.0)
    assert np.abs(x_q.astype(int)).max() <= 127
    assert np.all(np.abs(x_q.astype(int)).max(1) == 127)
    assert np.array_equal(rs, x_q.astype(np.int64).sum(1))
    # sign symmetry
    xq2, sx2, _, _ = oracle.rmsnorm_quant_act(-x, None, 0.0)
    assert np.array_equal(xq2, -x_q) and np.array_equal(sx2, s_x)
    # exact power-of-two scaling (eps = 0)
    for j in (-3, 4):
        xq3, sx3, _, _ = oracle.rmsnorm_quant_act(x * np.float32(2.0 ** j), None, 0.0)
        assert np.array_equal(xq3, x_q) and np.array_equal(sx3, s_x)
    # rows are independent
    perm = rng.permutation(16)
    xq4, sx4, _, _ = oracle.rmsnorm_quant_act(x[perm], None, 0.0)
    assert np.array_equal(xq4, x_q[perm]) and np.array_equal(sx4, s_x[perm])


@pytest.mark.parametrize("eps", [0.0, 1e-5])
def test_zero_activation_row(eps):
    x = np.zeros((2, 64), np.float32)
    x[1] = 1.0
    x_q, s_x, _, _ = oracle.rmsnorm_quant_act(x, None, eps)
    assert not x_q[0].any()
    assert s_x[0] == np.float32(127.0) / np.float32(1e-5)
    W = np.ones((3, 64), np.float32)
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    r = oracle.linear_forward(x, None, eps, W_p, s_w, 64)
    assert not r["y"][0].any()
    assert np.all(r["acc"][1] == 64 * 127)


def test_bf16_input_is_widened_exactly():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((4, 320)).astype(np.float32)
    xb = _bf16_bits(x)
    xw = oracle.bf16_bits_to_f32(xb)
    a = oracle.rmsnorm_quant_act(xb, None, 1e-5)
    b = oracle.rmsnorm_quant_act(xw, None, 1e-5)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# --------------------------------------------------------------- matmul

@pytest.mark.parametrize("seed", range(6))
def test_matmul_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    M, N = int(rng.integers(1, 33)), int(rng.integers(1, 65))
    K = 4 * int(rng.integers(1, 17))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s_w, _ = oracle.weight_scale(W)
    W_p, T = oracle.quantize_pack(W, s_w)
    x_q = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    acc = oracle.ternary_matmul(x_q, W_p, K)
    ref = x_q.astype(np.int64) @ T.astype(np.int64).T
    assert np.array_equal(acc, ref)
    assert np.abs(acc).max(initial=0) <= 128 * K
    cols = rng.permutation(N)[: max(1, N // 3)]
    assert np.array_equal(oracle.ternary_matmul(x_q, W_p, K, cols), ref[:, cols])


def test_matmul_is_x_times_w_transposed():
    # non-symmetric case: a transposed operand would give a different answer
    x_q = np.array([[1, 2, 3, 4]], np.int8)
    W = np.array([[1, 0, 0, 0], [0, 0, 0, -1], [1, 1, 0, 0]], np.float32)
    s_w, _ = oracle.weight_scale(W)  # mean|W| = 4/12 -> s_w = 3
    W_p, T = oracle.quantize_pack(W, s_w)
    assert T.tolist() == [[1, 0, 0, 0], [0, 0, 0, -1], [1, 1, 0, 0]]
    assert oracle.ternary_matmul(x_q, W_p, 4).tolist() == [[1, -4, 3]]


# -------------------------------------------------------------- dequant

def test_dequant_and_fake_quant_identity():
    case = workloads.CASES[0]
    x, W = workloads.tiny_inputs()
    s_w, _ = oracle.weight_scale(W)
    W_p, T = oracle.quantize_pack(W, s_w)
    r = oracle.linear_forward(x, None, workloads.DEFAULT_EPS, W_p, s_w, 256)
    denom = r["s_x"].astype(np.float64)[:, None] * np.float64(s_w)
    ref = r["acc"].astype(np.float64) / denom
    assert np.all(np.abs(r["y"] - ref) <= 2.0 ** -22 * np.abs(ref))
    # rescaled fake-quant product in fp64 equals the dequantized output
    fq = (r["x_q"].astype(np.float64) / r["s_x"].astype(np.float64)[:, None]) @ \
         (T.astype(np.float64) / np.float64(s_w)).T
    # (fq carries ~1e-16 of fp64 residue where acc == 0)
    assert np.all(np.abs(r["y"] - fq) <= 1e-6 * np.abs(fq) + 1e-12)
    yb = torch.from_numpy(r["y"]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["y_bf16"], yb)
    assert case.shapes[0] == (256, 512)


def test_forward_sign_symmetries():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    W = (rng.standard_normal((48, 256)) * 0.02).astype(np.float32)
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    Wn_p, _ = oracle.quantize_pack(-W, s_w)
    a = oracle.linear_forward(x, None, 1e-5, W_p, s_w, 256)
    b = oracle.linear_forward(-x, None, 1e-5, W_p, s_w, 256)
    c = oracle.linear_forward(x, None, 1e-5, Wn_p, s_w, 256)
    assert np.array_equal(a["y"], -b["y"])
    assert np.array_equal(a["y"], -c["y"])


def test_tiny_case_runs_in_ms():
    import time
    x, W = workloads.tiny_inputs()
    t0 = time.perf_counter()
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    r = oracle.linear_forward(x, None, workloads.DEFAULT_EPS, W_p, s_w, 256)
    assert time.perf_counter() - t0 < 2.0
    assert r["y"].shape == (16, 512)
