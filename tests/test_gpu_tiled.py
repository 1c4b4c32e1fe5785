"""Parity of the CUDA path on weights in the tiled layout.

The tiled layout only reorders the packed bytes (include/bitnet_b200.h,
bitnet_tile_weights).  The bytes are checked against a numpy restatement of
that documented order applied to the oracle's packed bytes; every forward
on tiled weights is checked against the oracle exactly like the row-major
path (x_q, s_x and the int32 accumulators bit for bit, fp32 y within 1e-6
relative, bf16 y within one ulp), and against the row-major path bit for
bit.
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


def retile(W_p, N, K):
    """The tiled order of the header, restated in numpy: tile (rb, c) of 128
    rows x 64 bytes, piece q of row r at r*64 + 16*(q ^ ((r >> 1) & 3))."""
    RB, KC = -(-N // 128), -(-K // 256)
    src = np.zeros((RB * 128, KC * 64), np.uint8)
    src[:N, :K // 4] = W_p
    out = np.zeros((RB, KC, 128, 4, 16), np.uint8)
    pieces = src.reshape(RB, 128, KC, 4, 16).transpose(0, 2, 1, 3, 4)  # rb, c, r, q, 16
    r = np.arange(128)[:, None]
    q = np.arange(4)[None, :]
    phys = q ^ ((r >> 1) & 3)                                           # [128, 4]
    for qq in range(4):
        out[:, :, np.arange(128), phys[:, qq], :] = pieces[:, :, :, qq, :]
    return out.reshape(-1)


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
    diff = np.abs(got.astype(np.int64) - y_ref_bf16.astype(np.int64))
    assert diff.max(initial=0) <= 1
    return float(np.mean(diff == 0))


def _weights_both(W):
    Wd = torch.from_numpy(W).cuda()
    W_p, s_w = tql.bitnet_quantize_pack_weights(Wd)
    del Wd
    return W_p, s_w, tql.bitnet_tile_weights(W_p)


@pytest.mark.parametrize("N,K", [(512, 256), (3200, 3200), (130, 8640), (1, 64), (129, 320),
                                 (257, 1088)])
def test_tiled_bytes_are_the_documented_order(N, K):
    rng = np.random.default_rng(N * 7 + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    ref_p, _ = oracle_weights(W)
    W_p, _, Wt = _weights_both(W)
    assert np.array_equal(W_p.cpu().numpy(), ref_p)
    assert Wt.data.numel() == tql.bitnet_tiled_weights_bytes(N, K) == retile(ref_p, N, K).size
    assert np.array_equal(Wt.data.cpu().numpy(), retile(ref_p, N, K))


def _forward_tiled_and_check(x, W, M, N, K, path, cols=None, gamma=None,
                             eps=workloads.DEFAULT_EPS,
                             y_dtypes=(torch.float32, torch.bfloat16)):
    W_p, s_w, Wt = _weights_both(W)
    ref_p, ref_s = oracle_weights(W)
    xd = x_to_device(x)
    gd = None if gamma is None else torch.from_numpy(gamma).cuda()
    ref = oracle.linear_forward(x, gamma, eps, ref_p, ref_s, K, cols)
    exact = []
    for ydt in y_dtypes:
        out = tql.bitnet_linear_forward_ex(xd, gd, eps, Wt, s_w, y_dtype=ydt, path=path)
        torch.cuda.synchronize()
        assert np.array_equal(out["x_q"].cpu().numpy(), ref["x_q"])
        assert np.array_equal(out["s_x"].cpu().numpy().view(np.uint32), ref["s_x"].view(np.uint32))
        acc = out["acc"].cpu().numpy()
        if cols is not None:
            acc = acc[:, cols]
        assert np.array_equal(acc, ref["acc"])
        exact.append(_check_y(out["y"], ref["y"], ref["y_bf16"], cols))
        # the same bits as the row-major weights through the plain forward
        y_rows = tql.bitnet_linear_forward(xd, gd, eps, W_p, s_w, y_dtype=ydt)
        torch.cuda.synchronize()
        if ydt == torch.bfloat16:
            assert torch.equal(y_rows.view(torch.int16), out["y"].view(torch.int16))
        else:
            assert torch.equal(y_rows, out["y"])
    return exact


@pytest.mark.parametrize("path", [tql.BITNET_PATH_AUTO, tql.BITNET_PATH_GEMM])
def test_tiled_tiny_case(path):
    x, W = workloads.tiny_inputs()
    exact = _forward_tiled_and_check(x, W, 16, 512, 256, path)
    assert min(exact) == 1.0


DECODE = [(c.index, si, M) for c in workloads.CASES[1:3] for si in range(len(c.shapes))
          for M in c.ms]


@pytest.mark.parametrize("ci,si,M", DECODE)
def test_tiled_decode_cases_full(ci, si, M):
    case = workloads.CASES[ci]
    K, N = case.shapes[si]
    x = workloads.activations(case, si, M)
    W = workloads.weights(case, si)
    _forward_tiled_and_check(x, W, M, N, K, tql.BITNET_PATH_AUTO, y_dtypes=(torch.bfloat16,))


LARGE = [(3, si, M) for si in range(2) for M in (512, 2048)] + \
        [(4, si, M) for si in range(2) for M in (1, 16, 64, 1024, 4096)]


@pytest.mark.parametrize("ci,si,M", LARGE)
def test_tiled_large_cases_sampled(ci, si, M):
    case = workloads.CASES[ci]
    K, N = case.shapes[si]
    x = workloads.activations(case, si, M)
    W = workloads.weights(case, si)
    cols = None if M <= 16 else sample_columns(N, 1024 if M <= 2048 else 256, seed=M + 7 * si)
    _forward_tiled_and_check(x, W, M, N, K, tql.BITNET_PATH_AUTO, cols=cols,
                             y_dtypes=(torch.bfloat16,))


RAGGED = [
    (1, 1, 64), (2, 33, 64), (3, 100, 192), (5, 31, 320), (7, 129, 1088), (9, 257, 8640),
    (16, 1000, 3200), (17, 130, 256), (63, 127, 576), (65, 255, 1216), (129, 300, 704),
    (200, 1, 128), (300, 520, 8640),
    # few rows, long K: several CTAs share one row block (partial slots)
    (1, 64, 16384), (4, 100, 20480), (13, 130, 32768), (16, 1, 65536),
    # many short row blocks per CTA
    (8, 40000, 256), (11, 9000, 512),
]


@pytest.mark.parametrize("M,N,K", RAGGED)
@pytest.mark.parametrize("path", [tql.BITNET_PATH_AUTO, tql.BITNET_PATH_GEMM])
def test_tiled_ragged_shapes(M, N, K, path):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    gamma = workloads.random_gamma(K)
    cols = None if N <= 4096 else sample_columns(N, 512, seed=N)
    _forward_tiled_and_check(x, W, M, N, K, path, gamma=gamma, cols=cols)


@pytest.mark.parametrize("M", [1, 16])
def test_tiled_grouped_mixed_layouts_and_shared_input(M):
    # Llama-3-8B decode projections: q/k/v share one input, gate/up another;
    # some weights tiled, some row-major; plus a tcgen05-sized problem.
    case = workloads.CASES[2]
    xq = workloads.activations(case, 0, M)
    xg = workloads.activations(case, 2, M)
    rng = np.random.default_rng(5 + M)
    xd = {id(xq): x_to_device(xq), id(xg): x_to_device(xg)}
    specs = [(0, xq, True), (1, xq, True), (1, xq, False), (2, xg, True), (2, xg, False),
             (3, None, True)]
    items, refs = [], []
    for j, (si, xh, tiled) in enumerate(specs):
        K, N = case.shapes[si]
        if xh is None:   # a prefill-sized problem on the tensor-core path
            xh = workloads._to_bf16_bits(rng.standard_normal((40, K)).astype(np.float32))
            xd[id(xh)] = x_to_device(xh)
        Mj = xh.shape[0]
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W_p, s_w, Wt = _weights_both(W)
        ref_p, ref_s = oracle_weights(W)
        ydt = torch.float32 if j % 2 else torch.bfloat16
        y = torch.empty((Mj, N), dtype=ydt, device="cuda")
        items.append((xd[id(xh)], None, workloads.DEFAULT_EPS, Wt if tiled else W_p, s_w, y))
        cols = None if Mj <= 16 else sample_columns(N, 256, seed=N)
        refs.append((oracle.linear_forward(xh, None, workloads.DEFAULT_EPS, ref_p, ref_s, K, cols),
                     cols))
    arr, count = tql.grouped_problems(items)
    nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ws.fill_(0xA5)   # contents on entry must not matter
    for _ in range(2):
        for it in items:
            it[5].fill_(0)
        tql.bitnet_linear_forward_grouped(items, workspace=ws)
        torch.cuda.synchronize()
        for it, (ref, cols) in zip(items, refs):
            _check_y(it[5], ref["y"], ref["y_bf16"], cols)


# Tiled problems of one token tile (M <= 8) and of two (M > 8) in one grouped
# call: one launch of the two-tile kernel in which single-token segments run
# on dp4a, 2..8-token segments on one MMA token tile and the rest on two.
# Ragged N and K, one-tile problems, both y dtypes.
MIXED_TILES = [
    [(1, 4096, 4096), (16, 4096, 4096), (1, 14336, 4096), (12, 4096, 1024)],
    [(16, 256, 128), (1, 8192, 4096)],
    [(9, 768, 300), (3, 1280, 1000), (1, 256, 130), (16, 2304, 520), (5, 512, 64)],
]


@pytest.mark.parametrize("ci", range(len(MIXED_TILES)))
def test_tiled_grouped_one_and_two_token_tiles(ci):
    rng = np.random.default_rng(31 + ci)
    items, refs = [], []
    for j, (M, K, N) in enumerate(MIXED_TILES[ci]):
        xh = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        _, s_w, Wt = _weights_both(W)
        ref_p, ref_s = oracle_weights(W)
        ydt = torch.float32 if j % 2 else torch.bfloat16
        y = torch.empty((M, N), dtype=ydt, device="cuda")
        items.append((x_to_device(xh), None, workloads.DEFAULT_EPS, Wt, s_w, y))
        refs.append(oracle.linear_forward(xh, None, workloads.DEFAULT_EPS, ref_p, ref_s, K))
    arr, count = tql.grouped_problems(items)
    nb = tql.bitnet_linear_forward_grouped_workspace_bytes(arr, count)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ws.fill_(0xA5)   # contents on entry must not matter
    for _ in range(2):
        for it in items:
            it[5].fill_(0)
        tql.bitnet_linear_forward_grouped(items, workspace=ws)
        torch.cuda.synchronize()
        for it, ref in zip(items, refs):
            _check_y(it[5], ref["y"], ref["y_bf16"])
    code, detail = tql.bitnet_device_status(reset=False)
    assert code == 0, (code, detail)


def test_tiled_workspace_garbage_on_entry():
    # Partial slots and counters: a workspace full of garbage must not
    # change the result (the counters are cleared by the quant launch).
    M, N, K = 16, 300, 32768
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W_p, s_w, Wt = _weights_both(W)
    xd = x_to_device(x)
    ws = torch.empty(tql.bitnet_linear_forward_workspace_bytes(M, N, K), dtype=torch.uint8,
                     device="cuda")
    ys = []
    for fill in (0x00, 0xFF, 0x5A):
        ws.fill_(fill)
        out = tql.bitnet_linear_forward_ex(xd, None, 1e-5, Wt, s_w, y_dtype=torch.float32,
                                           workspace=ws, debug=False)
        torch.cuda.synchronize()
        ys.append(out["y"].clone())
    ref_p, ref_s = oracle_weights(W)
    ref = oracle.linear_forward(x, None, 1e-5, ref_p, ref_s, K)
    for y in ys:
        _check_y(y, ref["y"], ref["y_bf16"])
        assert torch.equal(y, ys[0])


def test_no_device_failure_recorded_tiled():
    code, detail = tql.bitnet_device_status(reset=False)
    assert code == tql.BITNET_OK, detail


# ------------------------------------------------------- fused SwiGLU (decode)

def test_pair_tiled_bytes_interleave_two_tiled_layouts():
    rng = np.random.default_rng(21)
    N, K = 300, 1088
    Wg = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wu = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    pg, _, _ = _weights_both(Wg)
    pu, _, _ = _weights_both(Wu)
    pair = tql.bitnet_tile_weights_pair(pg, pu)
    tg = retile(pg.cpu().numpy(), N, K).reshape(-1, 8192)
    tu = retile(pu.cpu().numpy(), N, K).reshape(-1, 8192)
    want = np.stack([tg, tu], axis=1).reshape(-1)
    assert np.array_equal(pair.data.cpu().numpy(), want)


def _check_swiglu(y, ref_f32, ref_bf16):
    if y.dtype == torch.float32:
        got = y.cpu().numpy().astype(np.float64)
        err = np.abs(got - ref_f32)
        assert np.all(err <= 1e-6 * np.abs(ref_f32) + 1e-30), err.max()
    else:
        got = bf16_bits(y).astype(np.int64)
        assert np.abs(got - ref_bf16.astype(np.int64)).max(initial=0) <= 1


SWIGLU = [(2, 2, 1), (2, 2, 8), (2, 2, 16), (1, 1, 4), (None, None, 13)]


@pytest.mark.parametrize("ci,si,M", SWIGLU)
def test_swiglu_forward_matches_oracle(ci, si, M):
    rng = np.random.default_rng(17 + M)
    if ci is None:   # ragged: N and K tails, a gain vector
        N, K = 130, 8640
        x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        gamma = workloads.random_gamma(K)
    else:
        case = workloads.CASES[ci]
        K, N = case.shapes[si]
        x = workloads.activations(case, si, M)
        gamma = None
    Wg = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wu = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    pg, sg, _ = _weights_both(Wg)
    pu, su, _ = _weights_both(Wu)
    pair = tql.bitnet_tile_weights_pair(pg, pu)
    ref_pg, ref_sg = oracle_weights(Wg)
    ref_pu, ref_su = oracle_weights(Wu)
    ref = oracle.swiglu_forward(x, gamma, workloads.DEFAULT_EPS, ref_pg, ref_sg, ref_pu, ref_su,
                                K)
    xd = x_to_device(x)
    gd = None if gamma is None else torch.from_numpy(gamma).cuda()
    for ydt in (torch.float32, torch.bfloat16):
        for _ in range(2):
            y = tql.bitnet_swiglu_forward(xd, gd, workloads.DEFAULT_EPS, pair, sg, su, y_dtype=ydt)
            torch.cuda.synchronize()
            _check_swiglu(y, ref["y"].astype(np.float64), ref["y_bf16"])


def test_swiglu_rejects_prefill_sized_batches():
    rng = np.random.default_rng(3)
    N, K = 64, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    p, s, _ = _weights_both(W)
    pair = tql.bitnet_tile_weights_pair(p, p)
    x = x_to_device(workloads._to_bf16_bits(rng.standard_normal((17, K)).astype(np.float32)))
    with pytest.raises(tql.BitnetError):
        tql.bitnet_swiglu_forward(x, None, 1e-5, pair, s, s)


def test_concatenated_qkv_weights_in_one_buffer():
    # q, k and v tiled back to back in ONE buffer, read by one grouped call
    # that quantizes the shared input once (one quant and one matmul launch).
    case = workloads.CASES[2]
    M = 16
    x = workloads.activations(case, 0, M)
    rng = np.random.default_rng(8)
    shapes = [(4096, 4096), (4096, 1024), (4096, 1024)]
    sizes = [tql.bitnet_tiled_weights_bytes(N, K) for K, N in shapes]
    buf = torch.empty(sum(sizes), dtype=torch.uint8, device="cuda")
    xd = x_to_device(x)
    items, refs, off = [], [], 0
    for (K, N), nb in zip(shapes, sizes):
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W_p, s_w, _ = _weights_both(W)
        Wt = tql.bitnet_tile_weights(W_p, out=buf[off:off + nb])
        off += nb
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        items.append((xd, None, workloads.DEFAULT_EPS, Wt, s_w, y))
        ref_p, ref_s = oracle_weights(W)
        refs.append(oracle.linear_forward(x, None, workloads.DEFAULT_EPS, ref_p, ref_s, K))
    tql.bitnet_linear_forward_grouped(items)
    torch.cuda.synchronize()
    for it, ref in zip(items, refs):
        _check_y(it[5], ref["y"], ref["y_bf16"])


# The tcgen05 kernel on tiled weights for 16 < M <= 64 (split-K token tiles
# of 32 and 64): odd row-block counts, long K split over many CTAs, many
# short row blocks.
STREAM = [(17, 128, 256), (20, 300, 1088), (32, 4096, 4096), (33, 1000, 16384),
          (40, 129, 8192), (64, 4096, 4096), (64, 200, 65536), (48, 40000, 256)]


@pytest.mark.parametrize("M,N,K", STREAM)
def test_tcgen05_small_batch_tiled_shapes(M, N, K):
    rng = np.random.default_rng(M * 104729 + N * 131 + K)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    cols = None if N <= 4096 else sample_columns(N, 512, seed=N + M)
    exact = _forward_tiled_and_check(x, W, M, N, K, tql.BITNET_PATH_GEMM, cols=cols)
    assert min(exact) >= 0.0
