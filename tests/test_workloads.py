"""The seeded synthetic inputs follow their stated recipe (CPU only).

The recipe: W ~ N(0, sigma^2) with sigma = 0.02 (0.015 for the 70B sweep);
x ~ N(0, 1) with max(1, round(0.001 K)) outlier channels, the same for every
token, scaled by 20 (the per-feature outlier picture of the bitsandbytes
page, section on the outlier threshold), or a per-token scale exp(0.5 z) for
the prefill shapes; bf16 by round-to-nearest-even.  Sizes stay small so the
suite runs in seconds.
"""
import numpy as np
import pytest
import torch

from ternary_quantized_linear_b200 import workloads


@pytest.mark.parametrize("K,expected", [(3200, 3), (4096, 4), (8192, 8), (8640, 9),
                                        (14336, 14), (28672, 29), (256, 1)])
def test_outlier_channel_count(K, expected):
    assert max(1, int(round(0.001 * K))) == expected


def test_outlier_channels_per_case():
    for case in workloads.CASES:
        for si, (K, _) in enumerate(case.shapes):
            ch = workloads.outlier_channels(case, si, 1)
            if not case.outliers:
                assert ch is None
                continue
            assert len(ch) == max(1, int(round(0.001 * K)))
            assert len(np.unique(ch)) == len(ch)
            assert ch.min() >= 0 and ch.max() < K
            assert np.array_equal(ch, np.sort(ch))


def test_outlier_channels_are_scaled_by_20():
    case = workloads.CASE_BY_NAME["decode_bitnet3b"]
    si, M = 2, 16                                       # K = 8640: 9 outlier channels
    x = workloads.activations(case, si, M, f32=True)
    ch = workloads.outlier_channels(case, si, M)
    rest = np.setdiff1d(np.arange(x.shape[1]), ch)
    ratio = np.abs(x[:, ch]).mean() / np.abs(x[:, rest]).mean()
    assert 15.0 < ratio < 25.0                          # 20 x E|N(0,1)| over 144 draws
    # the same channels for every token: each row's largest entries sit there
    top = np.argsort(-np.abs(x), axis=1)[:, :1]
    assert np.isin(top, ch).mean() > 0.9


def test_activations_are_bf16_of_the_fp32_draw():
    case = workloads.CASE_BY_NAME["decode_llama3_8b"]
    x32 = workloads.activations(case, 0, 8, f32=True)
    bits = workloads.activations(case, 0, 8)
    assert bits.dtype == np.uint16 and bits.shape == x32.shape
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    # round to nearest even: the widened value is within half a bf16 ulp
    wide = (bits.astype(np.uint32) << 16).view(np.float32)
    ulp = np.abs(x32) * 2.0 ** -7
    assert np.all(np.abs(wide - x32) <= 0.5 * ulp + 1e-30)


def test_weight_sigma():
    case = workloads.CASE_BY_NAME["decode_bitnet3b"]
    W = workloads.weights(case, 0)
    assert W.dtype == np.float32 and W.shape == (3200, 3200)
    assert abs(W.std() / 0.02 - 1.0) < 5e-3
    assert abs(W.mean()) < 1e-4
    assert workloads.CASE_BY_NAME["sweep_70b"].sigma == 0.015


def test_prefill_tokens_have_lognormal_scale():
    case = workloads.CASE_BY_NAME["prefill_llama3_8b"]
    x = workloads.activations(case, 0, 512, f32=True)
    assert workloads.outlier_channels(case, 0, 512) is None
    log_rms = np.log(np.sqrt((x.astype(np.float64) ** 2).mean(axis=1)))
    assert abs(log_rms.std() / 0.5 - 1.0) < 0.15
    assert abs(log_rms.mean()) < 0.1


def test_draws_are_deterministic_and_distinct():
    case = workloads.CASE_BY_NAME["decode_bitnet3b"]
    a = workloads.activations(case, 0, 4)
    assert np.array_equal(a, workloads.activations(case, 0, 4))
    b = workloads.activations(case, 1, 4)          # same K, another shape: another stream
    assert not np.array_equal(a, b)
    c = workloads.activations(case, 0, 16)
    assert not np.array_equal(a, c[:4])
    x, W = workloads.tiny_inputs()
    assert x.dtype == np.float32 and x.shape == (16, 256) and W.shape == (512, 256)
    assert np.array_equal(W, workloads.weights(workloads.CASES[0], 0))
