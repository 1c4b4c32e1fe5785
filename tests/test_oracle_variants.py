"""Pins of the oracle's forward variants (no GPU): the SwiGLU of two BitLinear
outputs, the lambda-warmup fake-quant forward, BitDelta compression and its
multi-tenant forward, and group-wise scales.  Each function is checked
against something other than itself: closed forms, exact rational
arithmetic on hand-built cases, independent numpy fp64 computations of the
same definition, and the special cases where a variant reduces to the
already pinned per-tensor forward.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from ternary_quantized_linear_b200 import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def _ulp32(v):
    return float(np.spacing(np.float32(abs(v))))


# ---------------------------------------------------------------- SwiGLU

def test_silu_closed_forms():
    z = np.array([0.0, 1.0, -1.0, math.log(3.0), 30.0, -30.0, 2.0], np.float32)
    out, _ = oracle.swiglu(z, np.ones_like(z))
    exact = [0.0, 1.0 / (1.0 + math.exp(-1.0)), -1.0 / (1.0 + math.exp(1.0)),
             0.75 * float(np.float32(math.log(3.0))), 30.0 / (1.0 + math.exp(-30.0)),
             -30.0 / (1.0 + math.exp(30.0)), 2.0 / (1.0 + math.exp(-2.0))]
    for o, e in zip(out, exact):
        assert abs(float(o) - e) <= _ulp32(e) + 1e-45


def test_silu_odd_part_identity_and_linearity_in_up():
    # silu(z) - silu(-z) = z (sigma(z) + sigma(-z) = 1); the output is linear in up
    rng = np.random.default_rng(4)
    z = (rng.standard_normal(4096) * 4).astype(np.float32)
    a, _ = oracle.swiglu(z, np.ones_like(z))
    b, _ = oracle.swiglu(-z, np.ones_like(z))
    d = a.astype(np.float64) - b.astype(np.float64)
    assert np.all(np.abs(d - z) <= 4 * np.spacing(np.abs(z)) + 1e-30)
    u = (rng.standard_normal(4096)).astype(np.float32)
    o1, _ = oracle.swiglu(z, u)
    o2, _ = oracle.swiglu(z, (2 * u).astype(np.float32))
    assert np.array_equal(o2, (2 * o1).astype(np.float32))


def test_swiglu_forward_is_gate_and_up_forwards():
    x, W = workloads.tiny_inputs()
    Wu = W[::-1].copy()
    sg, _ = oracle.weight_scale(W)
    su, _ = oracle.weight_scale(Wu)
    Wg_p, _ = oracle.quantize_pack(W, sg)
    Wu_p, _ = oracle.quantize_pack(Wu, su)
    r = oracle.swiglu_forward(x, None, 1e-5, Wg_p, sg, Wu_p, su, 256)
    g = r["gate"]["y"].astype(np.float64)
    u = r["up"]["y"].astype(np.float64)
    ref = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
    assert np.array_equal(r["y"], ref)


# --------------------------------------------------- lambda-warmup forward

def test_warmup_lambda_schedule():
    assert oracle.warmup_lambda(0, 100) == 0.0
    assert oracle.warmup_lambda(25, 100) == 0.25
    assert oracle.warmup_lambda(100, 100) == 1.0
    assert oracle.warmup_lambda(250, 100) == 1.0


def _golden_4x64():
    """The hand-worked 4x4 case repeated 16 times along K (every row sum and
    scale is unchanged: mean |W| = 0.5, s_w = 2; each x row keeps its r and
    s_x = 64)."""
    with open(os.path.join(HERE, "golden", "bitlinear_4x4.json")) as f:
        gd = json.load(f)
    W = np.tile(np.array(gd["W"], np.float32), (1, 16))
    x = np.tile(np.array(gd["x"], np.float32), (1, 16))
    gamma = np.tile(np.array(gd["gamma"], np.float32), 16)
    return gd, x, W, gamma


def test_warmup_golden_half_lambda_exact():
    # lambda = 1/2 on the golden case: every operand is a small dyadic
    # rational, so the exact result (Fractions) must be reproduced exactly.
    gd, x, W, gamma = _golden_4x64()
    lam = 0.5
    r = oracle.warmup_forward(x, gamma, 0.0, W, lam)
    xq = np.tile(np.array(gd["x_q"], np.int64), (1, 16))
    T = np.tile(np.array(gd["T"], np.int64), (1, 16))
    rs = [Fraction(1), Fraction(1, 2), Fraction(1, 4), Fraction(2)]   # r of each row
    s_x, s_w = Fraction(64), Fraction(2)
    L = Fraction(1, 2)
    for m in range(4):
        xl = []
        for k in range(64):
            xn = Fraction(float(x[m, k])) * rs[m] * Fraction(float(gamma[k]))
            xt = Fraction(int(xq[m, k])) / s_x
            xl.append(xn + L * (xt - xn))
            assert Fraction(float(r["x_lam"][m, k])) == xl[k]
        for n in range(4):
            y = Fraction(0)
            for k in range(64):
                w = Fraction(float(W[n, k]))
                wl = w + L * (Fraction(int(T[n, k])) / s_w - w)
                y += xl[k] * wl
            assert Fraction(r["y"][m, n]) == y


def test_warmup_lambda_zero_is_the_full_precision_forward():
    rng = np.random.default_rng(11)
    M, N, K = 5, 37, 320
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    gamma = workloads.random_gamma(K)
    _, _, _, xn = oracle.rmsnorm_quant_act(x, gamma, 1e-5)
    ref = xn.astype(np.float64) @ W.astype(np.float64).T
    r = oracle.warmup_forward(x, gamma, 1e-5, W, 0.0)
    assert np.allclose(r["y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_warmup_lambda_one_is_the_quantized_forward():
    # lambda = 1: x_lam = x_q / s_x and W_lam = t / s_w, so the product is the
    # integer forward rescaled -- the same y as the inference path within
    # fp32 rounding of its two divisions.
    case = workloads.CASES[2]
    x = workloads.activations(case, 1, 8)
    W = workloads.weights(case, 1)[:300]
    K = W.shape[1]
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    inf = oracle.linear_forward(x, None, 1e-5, W_p, s_w, K)
    r = oracle.warmup_forward(x, None, 1e-5, W, 1.0)
    # x_q / s_x and t / s_w are each rounded to fp32 (2^-24 relative), the
    # inference quotient once (2^-24): the two agree within that bound,
    # relative to the sum of |products| (exact zeros of acc stay tiny).
    err = np.abs(r["y"] - inf["y"])
    assert np.all(err <= 2.0 ** -22 * (r["absdot"] + np.abs(inf["y"])))
    nz = inf["acc"] != 0
    assert (err[nz] / np.abs(inf["y"][nz])).max() <= 1e-6 or \
        np.all(err[nz] <= 2.0 ** -22 * r["absdot"][nz])


def test_warmup_bf16_operand_sum_stays_within_the_rounding_bound():
    rng = np.random.default_rng(12)
    x = workloads._to_bf16_bits(rng.standard_normal((3, 512)).astype(np.float32))
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    for lam in (0.0, 0.3, 1.0):
        r = oracle.warmup_forward(x, None, 1e-5, W, lam)
        # each bf16 operand is within 2^-9 relative of its fp32 value
        assert np.all(np.abs(r["y_b"] - r["y"]) <= 2.0 ** -7 * r["absdot"] + 1e-30)


# ------------------------------------------------------------- BitDelta

def _bf16(a):
    return workloads._to_bf16_bits(np.asarray(a, np.float32))


def _f32(bits):
    return oracle.bf16_bits_to_f32(bits)


def test_bitdelta_sign_zero_is_minus_one_and_packing_order():
    N, K = 2, 64
    base = np.zeros((N, K), np.float32)
    fine = np.zeros((N, K), np.float32)
    fine[0, 0] = 1.0      # +1 -> bit set
    fine[0, 33] = -2.0    # -1 -> bit clear
    fine[1, 31] = 0.5     # +1 in the top bit of word 0 of row 1
    signs, alpha, _ = oracle.bitdelta_compress(_bf16(base), _bf16(fine))
    assert signs.shape == (2, 2)
    assert signs[0, 0] == 1 and signs[0, 1] == 0
    assert signs[1, 0] == 1 << 31 and signs[1, 1] == 0
    assert alpha == np.float32(3.5 / (N * K))


def test_bitdelta_alpha_is_mean_abs_delta_and_l2_optimal():
    rng = np.random.default_rng(13)
    N, K = 48, 256
    base = _bf16(rng.standard_normal((N, K)) * 0.02)
    fine = _bf16(_f32(base) + rng.standard_normal((N, K)).astype(np.float32) * 0.002)
    signs, alpha, S = oracle.bitdelta_compress(base, fine)
    d = _f32(fine).astype(np.float64) - _f32(base).astype(np.float64)
    assert abs(S - math.fsum(np.abs(d).ravel())) <= 1e-13 * S
    assert alpha == np.float32(math.fsum(np.abs(d).ravel()) / (N * K))
    sgn = np.where(d > 0, 1.0, -1.0)
    err = lambda a: float(np.sum((d - a * sgn) ** 2))   # Eq. 3
    assert err(float(alpha)) < err(float(alpha) * 1.01)
    assert err(float(alpha)) < err(float(alpha) * 0.99)
    # unpack with the documented bit order
    bits = (signs[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    assert np.array_equal(np.where(bits.reshape(N, K) == 1, 1.0, -1.0), sgn)


def test_bitdelta_forward_is_the_reconstructed_matmul():
    rng = np.random.default_rng(14)
    B, N, K = 4, 40, 320
    base = _bf16(rng.standard_normal((N, K)) * 0.02)
    xs = _bf16(rng.standard_normal((B, K)))
    signs, alphas = [], []
    for b in range(B):
        fine = _bf16(_f32(base) + rng.standard_normal((N, K)).astype(np.float32) * 0.003)
        s, a, _ = oracle.bitdelta_compress(base, fine)
        signs.append(s)
        alphas.append(a)
    signs = np.stack(signs)
    alphas = np.array(alphas, np.float32)
    y, ad = oracle.bitdelta_forward(xs, base, signs, alphas)
    for b in range(B):
        bits = (signs[b][:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
        S = np.where(bits.reshape(N, K) == 1, 1.0, -1.0)
        Wrec = _f32(base).astype(np.float64) + float(alphas[b]) * S   # Eq. 1 + Eq. 6
        ref = _f32(xs[b]).astype(np.float64) @ Wrec.T
        assert np.all(np.abs(y[b] - ref) <= 1e-12 * ad[b])
    # tenants are independent: permuting them permutes the rows of y
    perm = [2, 0, 3, 1]
    y2, _ = oracle.bitdelta_forward(xs[perm], base, signs[perm], alphas[perm])
    assert np.array_equal(y2, y[perm])


# --------------------------------------------------------- group scales

def test_group_equal_to_k_is_the_per_tensor_forward():
    x, W = workloads.tiny_inputs()
    K = 256
    s = oracle.group_weight_scale(W, K)
    s_w, _ = oracle.weight_scale(W)
    assert s.shape == (1,) and s[0] == s_w
    W_p = oracle.group_quantize_pack(W, K, s)
    ref_p, _ = oracle.quantize_pack(W, s_w)
    assert np.array_equal(W_p, ref_p)
    g = oracle.group_linear_forward(x, None, 1e-5, W_p, s, K, K)
    ref = oracle.linear_forward(x, None, 1e-5, ref_p, s_w, K)
    assert np.array_equal(g["x_q"], ref["x_q"])
    assert np.array_equal(g["s_x"][:, 0], ref["s_x"])
    assert np.array_equal(g["acc"][:, :, 0], ref["acc"])
    assert np.array_equal(g["y"], ref["y"])


def test_group_scales_follow_each_group():
    rng = np.random.default_rng(15)
    N, K, gk = 64, 1024, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s = oracle.group_weight_scale(W, gk)
    for g in range(K // gk):
        blk = W[:, g * gk:(g + 1) * gk].astype(np.float64)
        mean = np.float32(math.fsum(np.abs(blk).ravel()) / blk.size)
        assert s[g] == np.float32(1.0) / mean
    # scaling group g by 2^g scales its scale by 2^-g and keeps every code
    W2 = W.copy()
    for g in range(K // gk):
        W2[:, g * gk:(g + 1) * gk] *= np.float32(2.0 ** g)
    s2 = oracle.group_weight_scale(W2, gk)
    assert np.array_equal(s2, (s * np.float32(2.0) ** -np.arange(K // gk)).astype(np.float32))
    assert np.array_equal(oracle.group_quantize_pack(W2, gk, s2),
                          oracle.group_quantize_pack(W, gk, s))


def test_group_forward_matches_the_fake_quant_identity():
    rng = np.random.default_rng(16)
    M, N, K, gk = 3, 48, 1024, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    x[:, :256] = workloads._to_bf16_bits(_f32(x[:, :256]) * np.float32(30.0))  # one loud group
    s = oracle.group_weight_scale(W, gk)
    W_p = oracle.group_quantize_pack(W, gk, s)
    r = oracle.group_linear_forward(x, None, 1e-5, W_p, s, K, gk)
    T = oracle.unpack(W_p, K).astype(np.float64)
    G = K // gk
    for g in range(G):
        q = r["x_q"][:, g * gk:(g + 1) * gk]
        assert np.all(np.abs(q).max(axis=1) == 127)      # each group reaches full range
    ref = np.zeros((M, N))
    for g in range(G):
        sl = slice(g * gk, (g + 1) * gk)
        ref += (r["x_q"][:, sl] / r["s_x"][:, g:g + 1].astype(np.float64)) @ \
               (T[:, sl] / float(s[g])).T
    rel = np.abs(r["y"] - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= 1e-6


# ----------------------------------------------- warm-up weights and backward

def test_warmup_weights_endpoints_and_agreement_with_the_forward():
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((24, 256)) * 0.02).astype(np.float32)
    w0, s0 = oracle.warmup_weights(W, 0.0)
    assert np.array_equal(w0.view(np.uint32), W.view(np.uint32))          # lambda = 0: W itself
    s_w, _ = oracle.weight_scale(W)
    assert np.float32(s0) == np.float32(s_w)
    # lambda = 1: every entry is a ternary level -1/s_w, 0 or 1/s_w, up to the
    # rounding of w + (t/s_w - w) (one fp32 subtraction, one addition)
    w1, _ = oracle.warmup_weights(W, 1.0)
    lev = np.float32(1.0) / np.float32(s_w)
    nearest = np.array([-lev, 0.0, lev], np.float32)
    dist = np.abs(w1[..., None] - nearest).min(-1)
    assert np.all(dist <= 4 * np.spacing(np.maximum(np.abs(W), lev)))
    # intermediate lambda: between W and its level, entry by entry
    wh, _ = oracle.warmup_weights(W, 0.5)
    lo = np.minimum(W, w1) - 4 * np.spacing(lev)
    hi = np.maximum(W, w1) + 4 * np.spacing(lev)
    assert np.all((wh >= lo) & (wh <= hi))
    # the forward's own W_lam: y(lambda) recomputed from the exported operands
    x = workloads._to_bf16_bits(rng.standard_normal((3, 256)).astype(np.float32))
    r = oracle.warmup_forward(x, None, 1e-5, W, 0.5)
    ref = r["x_lam"].astype(np.float64) @ wh.astype(np.float64).T
    assert np.allclose(r["y"], ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def _brute_bilinear(dy, xl, wl):
    """sum_{m,n} dy[m,n] sum_k xl[m,k] wl[n,k] by explicit loops (Fractions)."""
    M, N = dy.shape
    K = xl.shape[1]
    tot = Fraction(0)
    for m in range(M):
        for n in range(N):
            s = Fraction(0)
            for k in range(K):
                s += Fraction(float(xl[m, k])) * Fraction(float(wl[n, k]))
            tot += Fraction(float(dy[m, n])) * s
    return tot


def test_warmup_backward_is_the_derivative_of_the_bilinear_forward():
    # Small integers as bf16: every product and sum is exact.  The gradient
    # of f(X, W) = <dy, X W^T> in a direction E must equal the central
    # difference (exact for a bilinear f), and Euler's identity
    # <dy, y> = <dx, X> = <dW, W> must hold.
    rng = np.random.default_rng(22)
    M, N, K = 3, 4, 5
    to_bits = lambda a: workloads._to_bf16_bits(a.astype(np.float32))
    dy = to_bits(rng.integers(-3, 4, (M, N)))
    xl = to_bits(rng.integers(-4, 5, (M, K)))
    wl = to_bits(rng.integers(-2, 3, (N, K)))
    dx, dW = oracle.warmup_backward(dy, xl, wl)
    f = lambda X, Wm: _brute_bilinear(oracle.bf16_bits_to_f32(dy), X, Wm)
    X = oracle.bf16_bits_to_f32(xl)
    Wm = oracle.bf16_bits_to_f32(wl)
    E = rng.integers(-2, 3, (N, K)).astype(np.float32)
    Ex = rng.integers(-2, 3, (M, K)).astype(np.float32)
    dW_dir = (f(X, Wm + E) - f(X, Wm - E)) / 2
    dx_dir = (f(X + Ex, Wm) - f(X - Ex, Wm)) / 2
    assert Fraction(float((dW * E).sum())) == dW_dir
    assert Fraction(float((dx * Ex).sum())) == dx_dir
    y_dot = f(X, Wm)
    assert Fraction(float((dx * X).sum())) == y_dot
    assert Fraction(float((dW * Wm).sum())) == y_dot
