"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Integer and byte results (packed weights, x_q, int32 accumulators) must be
bit-exact.  Floating-point results: s_w and s_x are compared bit for bit
(both sides compute them with the same correctly rounded operations), the
fp32 output within max relative error 1e-6 and the bf16 output within one
bf16 ulp -- in practice both match exactly, and the tests also count exact
matches.  Large problems compare every x_q / s_x / packed byte and a seeded
sample of output columns (all rows) that the oracle computes one by one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import ternary_quantized_linear_b200 as tql
from ternary_quantized_linear_b200 import build as tql_build
from ternary_quantized_linear_b200 import workloads

from _util import bf16_bits, oracle_weights, sample_columns, x_to_device

pytestmark = pytest.mark.gpu

FP32_RTOL = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _setup():
    tql_build.build()
    tql.load_library()
    oracle.set_threads(os.cpu_count() or 1)
    torch.cuda.set_device(0)
    yield


def _dev_weights(W_np):
    W = torch.from_numpy(W_np).cuda()
    W_p, s_w = tql.bitnet_quantize_pack_weights(W)
    return W_p, s_w


def _check_y(y_dev, y_ref_f32, y_ref_bf16, cols=None):
    if y_dev.dtype == torch.float32:
        got = y_dev.cpu().numpy()
        if cols is not None:
            got = got[:, cols]
        err = np.abs(got.astype(np.float64) - y_ref_f32) / np.maximum(np.abs(y_ref_f32), 1e-30)
        err[y_ref_f32 == 0] = np.abs(got[y_ref_f32 == 0])
        assert err.max(initial=0.0) <= FP32_RTOL
        return float(np.mean(got == y_ref_f32))
    got = bf16_bits(y_dev)
    if cols is not None:
        got = got[:, cols]
    # one bf16 ulp == adjacent bit patterns of the same sign
    diff = np.abs(got.astype(np.int64) - y_ref_bf16.astype(np.int64))
    assert diff.max(initial=0) <= 1
    return float(np.mean(diff == 0))


# ------------------------------------------------------------- weights

WEIGHT_SHAPES = [(c.index, si) for c in workloads.CASES for si in range(len(c.shapes))]


@pytest.mark.parametrize("ci,si", WEIGHT_SHAPES)
def test_weight_quant_pack_bit_exact(ci, si):
    case = workloads.CASES[ci]
    W = workloads.weights(case, si)
    W_p, s_w = _dev_weights(W)
    ref_p, ref_s = oracle_weights(W)
    assert s_w.cpu().numpy()[0].tobytes() == np.float32(ref_s).tobytes()
    assert np.array_equal(W_p.cpu().numpy(), ref_p)


def test_weight_quant_edge_values():
    # exact ties, zeros and a tiny-magnitude matrix (scale floor)
    W = np.zeros((32, 64), np.float32)
    W[0, :4] = [0.25, -0.25, 0.75, -0.75]
    W[1, :4] = [0.5, -0.5, 1.0, -1.0]
    W_p, s_w = _dev_weights(W)
    ref_p, ref_s = oracle_weights(W)
    assert s_w.item() == float(ref_s)
    assert np.array_equal(W_p.cpu().numpy(), ref_p)
    tiny = np.full((16, 64), 1e-9, np.float32)
    W_p, s_w = _dev_weights(tiny)
    ref_p, ref_s = oracle_weights(tiny)
    assert s_w.item() == float(ref_s) == float(np.float32(1) / np.float32(1e-5))
    assert np.array_equal(W_p.cpu().numpy(), ref_p)


# --------------------------------------------------------- activations

ACT_CASES = [(0, 0, 16)] + [(c.index, si, M) for c in workloads.CASES[1:]
                            for si in range(len(c.shapes)) for M in c.ms if M <= 2048]


@pytest.mark.parametrize("ci,si,M", ACT_CASES)
def test_act_quant_bit_exact(ci, si, M):
    case = workloads.CASES[ci]
    x = workloads.activations(case, si, M)
    xd = x_to_device(x)
    x_q, s_x = tql.bitnet_rmsnorm_quant_act(xd, None, workloads.DEFAULT_EPS)
    rq, rs, _, _ = oracle.rmsnorm_quant_act(x, None, workloads.DEFAULT_EPS)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(x_q.cpu().numpy(), rq)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("eps", [0.0, 1e-5, 1e-2])
def test_act_quant_gamma_eps_zero_rows(dtype, eps):
    rng = np.random.default_rng(5)
    K = 4096 + 64 * 7
    x = rng.standard_normal((9, K)).astype(np.float32)
    x[2] = 0.0                  # all-zero row
    x[3] *= 1e-3
    x[4, 100] = 3.0e3           # one huge channel
    x[5] = np.float32(2.0 ** -10)
    if dtype == "bf16":
        x = workloads._to_bf16_bits(x)
    gamma = workloads.random_gamma(K)
    xd = x_to_device(x)
    x_q, s_x = tql.bitnet_rmsnorm_quant_act(xd, torch.from_numpy(gamma).cuda(), eps)
    rq, rs, _, _ = oracle.rmsnorm_quant_act(x, gamma, eps)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(x_q.cpu().numpy(), rq)


# ------------------------------------------------------------- forward

def _forward_and_check(x, W, M, N, K, path, cols=None, gamma=None, eps=workloads.DEFAULT_EPS,
                       y_dtypes=(torch.float32, torch.bfloat16)):
    W_p, s_w = _dev_weights(W)
    ref_p, ref_s = oracle_weights(W)
    assert np.array_equal(W_p.cpu().numpy(), ref_p)
    xd = x_to_device(x)
    gd = None if gamma is None else torch.from_numpy(gamma).cuda()
    ref = oracle.linear_forward(x, gamma, eps, ref_p, ref_s, K, cols)
    exact = []
    for ydt in y_dtypes:
        out = tql.bitnet_linear_forward_debug(xd, gd, eps, W_p, s_w, y_dtype=ydt, path=path)
        torch.cuda.synchronize()
        assert np.array_equal(out["x_q"].cpu().numpy(), ref["x_q"])
        assert np.array_equal(out["s_x"].cpu().numpy().view(np.uint32), ref["s_x"].view(np.uint32))
        acc = out["acc"].cpu().numpy()
        if cols is not None:
            acc = acc[:, cols]
        assert np.array_equal(acc, ref["acc"])
        exact.append(_check_y(out["y"], ref["y"], ref["y_bf16"], None if cols is None else cols))
        # the plain forward gives the same bits as the debug one
        y2 = tql.bitnet_linear_forward(xd, gd, eps, W_p, s_w, y_dtype=ydt)
        torch.cuda.synchronize()
        # (whichever path the plain call picks: both paths give identical bits)
        assert torch.equal(y2.view(torch.int16) if ydt == torch.bfloat16 else y2,
                           out["y"].view(torch.int16) if ydt == torch.bfloat16 else out["y"])
    return exact


@pytest.mark.parametrize("path", [tql.BITNET_PATH_AUTO, tql.BITNET_PATH_GEMV,
                                  tql.BITNET_PATH_GEMM])
def test_tiny_case_forward(path):
    x, W = workloads.tiny_inputs()
    exact = _forward_and_check(x, W, 16, 512, 256, path)
    assert min(exact) == 1.0


DECODE = [(c.index, si, M) for c in workloads.CASES[1:3] for si in range(len(c.shapes))
          for M in c.ms]


@pytest.mark.parametrize("ci,si,M", DECODE)
def test_decode_cases_full(ci, si, M):
    case = workloads.CASES[ci]
    K, N = case.shapes[si]
    x = workloads.activations(case, si, M)
    W = workloads.weights(case, si)
    _forward_and_check(x, W, M, N, K, tql.BITNET_PATH_AUTO, y_dtypes=(torch.bfloat16,))


@pytest.mark.parametrize("ci,si,M", [(1, 1, 16), (2, 3, 8), (2, 1, 1)])
def test_decode_paths_agree(ci, si, M):
    case = workloads.CASES[ci]
    K, N = case.shapes[si]
    x = workloads.activations(case, si, M)
    W = workloads.weights(case, si)
    _forward_and_check(x, W, M, N, K, tql.BITNET_PATH_GEMM, y_dtypes=(torch.float32,))


LARGE = [(3, si, M) for si in range(2) for M in (512, 2048, 8192)] + \
        [(4, si, M) for si in range(2) for M in (1, 16, 64, 1024, 4096)]


@pytest.mark.parametrize("ci,si,M", LARGE)
def test_large_cases_sampled(ci, si, M):
    case = workloads.CASES[ci]
    K, N = case.shapes[si]
    x = workloads.activations(case, si, M)
    W = workloads.weights(case, si)
    # 1024 sampled columns (plus tile edges) up to 2048 tokens, 256 beyond
    cols = None if M <= 16 else sample_columns(N, 1024 if M <= 2048 else 256, seed=M + 7 * si)
    _forward_and_check(x, W, M, N, K, tql.BITNET_PATH_AUTO, cols=cols,
                       y_dtypes=(torch.bfloat16,))


RAGGED = [
    # (M, N, K): tails on every axis, tile-boundary and minimum sizes
    (1, 1, 64), (2, 33, 64), (3, 100, 192), (5, 31, 320), (7, 129, 1088), (9, 257, 8640),
    (16, 1000, 3200), (17, 130, 256), (63, 127, 576), (65, 255, 1216), (129, 300, 704),
    (200, 1, 128), (300, 520, 8640),
    # few rows, long K: the decode matmul splits row blocks across CTAs
    (1, 64, 16384), (4, 100, 20480), (13, 130, 32768),
]


@pytest.mark.parametrize("M,N,K", RAGGED)
@pytest.mark.parametrize("path", [tql.BITNET_PATH_AUTO, tql.BITNET_PATH_GEMM])
def test_ragged_shapes(M, N, K, path):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    gamma = workloads.random_gamma(K)
    _forward_and_check(x, W, M, N, K, path, gamma=gamma)


def test_matmul_debug_entry_extreme_values():
    # x_q at the int8 extremes, every code pattern: exercises sign handling and |acc| ~ 127 K
    rng = np.random.default_rng(9)
    for (M, N, K) in [(4, 64, 256), (16, 96, 4096), (40, 200, 1024)]:
        x_q = rng.choice(np.array([-128, -127, 127, 0, 1, -1], np.int8), size=(M, K))
        x_q[0] = 127
        x_q[1 % M] = -128
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W[0] = 1.0
        W[1] = -1.0
        W_p, _ = _dev_weights(W)
        for path in (tql.BITNET_PATH_AUTO, tql.BITNET_PATH_GEMM):
            acc = tql.bitnet_ternary_matmul_i32(torch.from_numpy(x_q).cuda(), W_p, path=path)
            ref = oracle.ternary_matmul(x_q, W_p.cpu().numpy(), K)
            assert np.array_equal(acc.cpu().numpy(), ref)


def test_empty_batch_is_a_no_op():
    W_p = torch.zeros((64, 64), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((1,), device="cuda")
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    y = tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w)
    assert y.shape == (0, 64)


def test_workspace_is_left_zeroed_and_runs_are_deterministic():
    case = workloads.CASES[2]
    si, M = 3, 16
    K, N = case.shapes[si]
    x = x_to_device(workloads.activations(case, si, M))
    W_p, s_w = _dev_weights(workloads.weights(case, si))
    nb = tql.bitnet_linear_forward_workspace_bytes(M, N, K)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    y1 = tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w, workspace=ws)
    y2 = tql.bitnet_linear_forward(x, None, 1e-5, W_p, s_w, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    # split-K partials and counters are back to zero (x_q / scales may remain)
    # layout: x_q [M*K] | s_x [4M] | rowsum [4M] | partials | counters, each 256-aligned
    acc_off = ((M * K + 255) // 256) * 256 + 2 * ((4 * M + 255) // 256) * 256
    assert int(ws[acc_off:].count_nonzero()) == 0


def test_bounded_wait_reports_timeout():
    tql.bitnet_device_status(reset=True)
    tql.bitnet_selftest_bounded_wait(2_000_000)  # 2 ms, on a barrier nothing completes
    code, detail = tql.bitnet_device_status(reset=True)
    assert code == tql.BITNET_ERR_TIMEOUT and detail == 6
    code, detail = tql.bitnet_device_status(reset=False)
    assert code == tql.BITNET_OK and detail == 0
    # the context is still usable afterwards
    x, W = workloads.tiny_inputs()
    _forward_and_check(x, W, 16, 512, 256, tql.BITNET_PATH_GEMM, y_dtypes=(torch.float32,))


def test_no_device_failure_recorded():
    code, detail = tql.bitnet_device_status(reset=False)
    assert code == tql.BITNET_OK, detail


# ------------------------------------------------------------- grouped

def _grouped_items(case, extra=()):
    items, meta = [], []
    packed = {}
    for si, K, N, M in workloads.all_problems(case):
        if si not in packed:
            packed[si] = (workloads.weights(case, si),) + _dev_weights(workloads.weights(case, si))
        xh = workloads.activations(case, si, M)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        items.append((x_to_device(xh), None, workloads.DEFAULT_EPS, packed[si][1], packed[si][2], y))
        meta.append((xh, packed[si][0], K, N, M))
    for (M, N, K, ydt) in extra:
        rng = np.random.default_rng(M * 13 + N)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        xh = rng.standard_normal((M, K)).astype(np.float32)
        W_p, s_w = _dev_weights(W)
        y = torch.empty((M, N), dtype=ydt, device="cuda")
        items.append((x_to_device(xh), None, workloads.DEFAULT_EPS, W_p, s_w, y))
        meta.append((xh, W, K, N, M))
    return items, meta


@pytest.mark.parametrize("ci", [1, 2])
@pytest.mark.parametrize("split", [False, True])
def test_grouped_forward_matches_single_calls_and_oracle(ci, split):
    case = workloads.CASES[ci]
    # plus an fp32 decode problem, a prefill-sized one (tensor-core path) and an empty one
    items, meta = _grouped_items(case, extra=[(5, 96, 320, torch.float32),
                                              (40, 300, 512, torch.bfloat16),
                                              (0, 64, 256, torch.bfloat16)])
    if split:
        ws = torch.empty(1 << 26, dtype=torch.uint8, device="cuda")
        tql.bitnet_linear_forward_grouped(items, workspace=ws, phases=tql.BITNET_PHASE_QUANTIZE)
        tql.bitnet_linear_forward_grouped(items, workspace=ws, phases=tql.BITNET_PHASE_MATMUL)
    else:
        tql.bitnet_linear_forward_grouped(items)
    torch.cuda.synchronize()
    for (x, g, eps, W_p, s_w, y), (xh, W, K, N, M) in zip(items, meta):
        if M == 0:
            continue
        y1 = tql.bitnet_linear_forward(x, g, eps, W_p, s_w, y_dtype=y.dtype)
        torch.cuda.synchronize()
        if y.dtype == torch.bfloat16:
            assert torch.equal(y.view(torch.int16), y1.view(torch.int16))
        else:
            assert torch.equal(y, y1)
        ref_p, ref_s = oracle_weights(W)
        cols = None if N <= 4096 else sample_columns(N, 256, seed=N)
        ref = oracle.linear_forward(xh, None, eps, ref_p, ref_s, K, cols)
        _check_y(y, ref["y"], ref["y_bf16"], cols)


def test_grouped_rejects_bad_problem_and_queues_nothing():
    case = workloads.CASES[1]
    items, _ = _grouped_items(case)
    for it in items:
        it[5].fill_(0)
    bad = list(items)
    x, g, eps, W_p, s_w, y = bad[4]
    bad[4] = (x, g, -1.0, W_p, s_w, y)  # eps < 0
    with pytest.raises(tql.BitnetError):
        tql.bitnet_linear_forward_grouped(bad)
    torch.cuda.synchronize()
    assert all(int(it[5].count_nonzero()) == 0 for it in items)


@pytest.mark.parametrize("M", [1, 13])
def test_grouped_shared_input_and_repeated_calls(M):
    # q/k/v- and gate/up-style problems read the same x (one quantization is
    # shared); the call is repeated with the same problems (cached plan) and
    # then with new output buffers (a different plan): every result must be
    # the single-call result.
    rng = np.random.default_rng(77 + M)
    K = 1024
    x = x_to_device(workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)))
    x2 = x_to_device(workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)))
    gamma = torch.from_numpy(workloads.random_gamma(K)).cuda()
    mats = []
    for N in (1024, 256, 256, 2816, 2816):
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        mats.append(_dev_weights(W))

    def items_for(outs):
        its = []
        for j, ((W_p, s_w), y) in enumerate(zip(mats, outs)):
            xin, g = (x, gamma) if j < 3 else (x2, None)
            its.append((xin, g, 1e-5, W_p, s_w, y))
        return its

    def fresh():
        return [torch.empty((M, W_p.shape[0]), dtype=torch.bfloat16, device="cuda")
                for W_p, _ in mats]

    ys = fresh()
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        for y in ys:
            y.fill_(0)
        tql.bitnet_linear_forward_grouped(items_for(ys), workspace=ws)
    ys2 = fresh()
    tql.bitnet_linear_forward_grouped(items_for(ys2), workspace=ws)
    torch.cuda.synchronize()
    for j, (W_p, s_w) in enumerate(mats):
        xin, g = (x, gamma) if j < 3 else (x2, None)
        y1 = tql.bitnet_linear_forward(xin, g, 1e-5, W_p, s_w, y_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(ys[j].view(torch.int16), y1.view(torch.int16))
        assert torch.equal(ys2[j].view(torch.int16), y1.view(torch.int16))


def test_epilogue_division_matches_ieee_division():
    # The decode epilogue divides through a correctly rounded reciprocal and
    # two residual corrections; it must equal an IEEE binary32 division
    # (numpy on the host) for every value the dequant can see: integer
    # numerators up to 2^27 and divisors from products of scales, plus
    # significands at the edges (all ones, powers of two, near-midpoint
    # quotients) and random finite floats.
    rng = np.random.default_rng(2024)
    n = 1 << 22
    a_int = rng.integers(-(1 << 27), 1 << 27, n).astype(np.float32)
    sx = (127.0 / rng.uniform(1e-3, 300.0, n)).astype(np.float32)
    sw = rng.uniform(1.0, 400.0, n).astype(np.float32)
    b_prod = (sx * sw).astype(np.float32)
    ones = np.float32(2.0 ** 24 - 1) * np.power(np.float32(2.0), rng.integers(-30, 8, n).astype(np.float32))
    pow2 = np.power(np.float32(2.0), rng.integers(-20, 20, n).astype(np.float32))
    rnd_a = (rng.standard_normal(n) * np.exp(rng.uniform(-20, 20, n))).astype(np.float32)
    rnd_b = np.exp(rng.uniform(-20, 20, n)).astype(np.float32)
    a_mid = ((rng.integers(1, 1 << 24, n) * 2 + 1) * np.float32(0.5)).astype(np.float32)
    cases = [(a_int, b_prod), (a_int, ones.astype(np.float32)), (a_int, pow2.astype(np.float32)),
             (rnd_a, rnd_b), (a_mid, np.float32(3.0) * pow2.astype(np.float32)),
             (np.zeros(n, np.float32), b_prod)]
    for a, b in cases:
        ref = (a / b).astype(np.float32)
        assert np.all(np.isfinite(ref))
        q = tql.bitnet_selftest_divide(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
        torch.cuda.synchronize()
        got = q.cpu().numpy()
        bad = np.nonzero(got.view(np.uint32) != ref.view(np.uint32))[0]
        assert bad.size == 0, (a[bad[:5]], b[bad[:5]], got[bad[:5]], ref[bad[:5]])


@pytest.mark.parametrize("M", [1, 16])
def test_grouped_shared_quantization_matches_oracle(M):
    # q/k/v read one x and gate/up another (Llama-3-8B decode shapes): the
    # grouped call quantizes each distinct input once and the matmuls share
    # it.  Every output is compared with the oracle element by element, in
    # fp32 (<= 1e-6 relative) and bf16 (<= 1 ulp).
    case = workloads.CASES[2]
    xq = workloads.activations(case, 0, M)   # 4096 wide: the q/k/v input
    xg = workloads.activations(case, 2, M)   # 4096 wide: the gate/up input
    shapes = [(0, xq), (1, xq), (1, xq), (2, xg), (2, xg)]   # q, k, v, gate, up
    rng = np.random.default_rng(31 + M)
    items, refs = [], []
    xd = {id(xq): x_to_device(xq), id(xg): x_to_device(xg)}
    for j, (si, xh) in enumerate(shapes):
        K, N = case.shapes[si]
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W_p, s_w = _dev_weights(W)
        ref_p, ref_s = oracle_weights(W)
        ydt = torch.float32 if j % 2 == 0 else torch.bfloat16
        y = torch.empty((M, N), dtype=ydt, device="cuda")
        items.append((xd[id(xh)], None, workloads.DEFAULT_EPS, W_p, s_w, y))
        refs.append(oracle.linear_forward(xh, None, workloads.DEFAULT_EPS, ref_p, ref_s, K))
    arr, count = tql.grouped_problems(items)
    nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for _ in range(2):   # the second call replays the cached plan
        for it in items:
            it[5].fill_(0)
        tql.bitnet_linear_forward_grouped(items, workspace=ws)
        torch.cuda.synchronize()
        for it, ref in zip(items, refs):
            exact = _check_y(it[5], ref["y"], ref["y_bf16"])
            assert exact == 1.0


def test_default_workspace_is_per_stream():
    # Two side streams with no ordering between them, both using the
    # binding's default workspace: each must get its own buffer, and both
    # results must match the oracle.
    case = workloads.CASES[2]
    outs, refs = [], []
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    jobs = []
    for j, si in enumerate((3, 0)):
        K, N = case.shapes[si]
        xh = workloads.activations(case, si, 16)
        W = workloads.weights(case, si)
        W_p, s_w = _dev_weights(W)
        ref_p, ref_s = oracle_weights(W)
        refs.append(oracle.linear_forward(xh, None, workloads.DEFAULT_EPS, ref_p, ref_s, K))
        jobs.append((x_to_device(xh), W_p, s_w))
    torch.cuda.synchronize()
    for _ in range(3):
        outs = []
        for (x, W_p, s_w), st in zip(jobs, streams):
            with torch.cuda.stream(st):
                outs.append(tql.bitnet_linear_forward(x, None, workloads.DEFAULT_EPS, W_p, s_w,
                                                      y_dtype=torch.float32))
        torch.cuda.synchronize()
        for y, ref in zip(outs, refs):
            _check_y(y, ref["y"], ref["y_bf16"])


def test_division_outside_the_fast_range_is_ieee():
    # Subnormal and zero divisors, quotients that overflow, numerators near
    # the range ends: the epilogue division falls back to IEEE division there.
    a = np.array([1.0, -3.0, 1e30, 7.0, 1e-30, 3.0e38, 2.0, 0.0, 5.0, -1e20],
                 np.float32)
    b = np.array([1e-40, 1e-39, 1e-10, 0.0, 3.0, 0.5, 3.0e38, 1e-40, np.float32(2.0 ** -126),
                  1e-20], np.float32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        ref = (a / b).astype(np.float32)
    q = tql.bitnet_selftest_divide(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    torch.cuda.synchronize()
    got = q.cpu().numpy()
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), (a[~same], b[~same], got[~same], ref[~same])


@pytest.mark.parametrize("split", [False, True])
def test_grouped_tensor_core_problems_share_the_quant_launch(split):
    # Larger problems are quantized by the grouped launch too: two M = 64
    # problems on one input (split-K partials, one shared quantization), an
    # M = 300 problem, and a decode problem; every output must equal the
    # single-call forward bit for bit and the oracle within the usual bar.
    rng = np.random.default_rng(404)
    K = 1024
    x64 = workloads._to_bf16_bits(rng.standard_normal((64, K)).astype(np.float32))
    x300 = workloads._to_bf16_bits(rng.standard_normal((300, K)).astype(np.float32))
    x1 = workloads._to_bf16_bits(rng.standard_normal((1, K)).astype(np.float32))
    d64, d300, d1 = x_to_device(x64), x_to_device(x300), x_to_device(x1)
    specs = [(x64, d64, 640), (x64, d64, 200), (x300, d300, 384), (x1, d1, 520)]
    items, meta = [], []
    for xh, xd, N in specs:
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W_p, s_w = _dev_weights(W)
        y = torch.empty((xh.shape[0], N), dtype=torch.bfloat16, device="cuda")
        items.append((xd, None, workloads.DEFAULT_EPS, W_p, s_w, y))
        meta.append((xh, W, N))
    if split:
        ws = torch.empty(1 << 26, dtype=torch.uint8, device="cuda")
        ws.fill_(0x5A)
        tql.bitnet_linear_forward_grouped(items, workspace=ws, phases=tql.BITNET_PHASE_QUANTIZE)
        tql.bitnet_linear_forward_grouped(items, workspace=ws, phases=tql.BITNET_PHASE_MATMUL)
    else:
        tql.bitnet_linear_forward_grouped(items)
    torch.cuda.synchronize()
    for (xd, g, eps, W_p, s_w, y), (xh, W, N) in zip(items, meta):
        y1 = tql.bitnet_linear_forward(xd, g, eps, W_p, s_w, y_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y1.view(torch.int16))
        ref_p, ref_s = oracle_weights(W)
        ref = oracle.linear_forward(xh, None, eps, ref_p, ref_s, K)
        _check_y(y, ref["y"], ref["y_bf16"])
