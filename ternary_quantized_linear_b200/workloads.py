"""Seeded synthetic inputs for the BitLinear forward (shapes and value recipes).

This module only draws random numbers and builds shapes; it holds none of the
method's arithmetic (no normalisation, no quantization, no packing).  Both the
CUDA path's tests/benchmark and the CPU oracle consume exactly these arrays.

Recipes (the pages measure on no public kernel benchmark; these shapes follow
the model families the pages talk about -- BitNet b1.58 3B, Llama-3-8B
fine-tuned to 1.58 bit, and a 70B-class model):

* weights  W [N, K] fp32 ~ N(0, sigma^2), sigma = 0.02 (0.015 for the 70B sweep)
* activations x [M, K] ~ N(0, 1) drawn in fp32, then
    - outlier channels: k_out = max(1, round(0.001 K)) channels, the same for
      every token, multiplied by 20 (the per-feature outlier picture of the
      bitsandbytes LLM.int8() page);
    - or a per-token scale exp(0.5 z_m), z_m ~ N(0,1) (prefill shapes);
  and rounded to bf16 (round to nearest even) except for the tiny case,
  which stays fp32.
* gamma = 1, eps = 1e-5.

Generators: numpy PCG64.  The tiny case draws x then W from PCG64(0).  Every
other case uses PCG64 seeded with the integer tuple
(case_index, shape_index, stream, ...): stream 0 for W, stream 1 (+ M) for x.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class Case:
    index: int                         # position in CASES
    name: str
    shapes: Tuple[Tuple[int, int], ...]  # (K, N) pairs, y = x W^T with W [N,K]
    ms: Tuple[int, ...]                # token counts
    sigma: float
    outliers: bool
    token_lognormal: bool
    x_dtype: str                       # "f32" or "bf16"
    description: str = ""


CASES: List[Case] = [
    Case(0, "tiny", ((256, 512),), (16,), 0.02, False, False, "f32",
         "x [16 x 256] fp32 N(0,1), W [512 x 256] N(0,0.02^2); fp32 output; seed 0"),
    Case(1, "decode_bitnet3b", ((3200, 3200), (3200, 8640), (8640, 3200)), (1, 4, 16),
         0.02, True, False, "bf16",
         "decode GEMV, BitNet-3B-shaped (hidden 3200, ffn 8640), bf16 acts + 0.1% x20 outlier channels"),
    Case(2, "decode_llama3_8b", ((4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)),
         (1, 8, 16), 0.02, True, False, "bf16",
         "decode GEMV, Llama-3-8B-shaped q/o, k/v, gate/up, down; bf16 acts + outliers"),
    Case(3, "prefill_llama3_8b", ((4096, 14336), (14336, 4096)), (512, 2048, 8192),
         0.02, False, True, "bf16",
         "prefill GEMM, Llama-3-8B FFN shapes; bf16 acts with per-token LogNormal(0,0.5) scale"),
    Case(4, "sweep_70b", ((8192, 28672), (28672, 8192)), (1, 16, 64, 1024, 4096),
         0.015, True, False, "bf16",
         "70B-shaped sweep (hidden 8192, ffn 28672), bf16 acts + outliers, W sigma 0.015"),
]

CASE_BY_NAME = {c.name: c for c in CASES}

DEFAULT_EPS = 1e-5


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(list(key)))


def _to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) via torch's CPU cast; return bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def tiny_inputs():
    """The tiny case: (x fp32 [16,256], W fp32 [512,256]) from PCG64(0), x drawn first."""
    rng = np.random.Generator(np.random.PCG64(0))
    x = rng.standard_normal((16, 256), dtype=np.float32)
    W = (rng.standard_normal((512, 256), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    return x, W


def weights(case: Case, shape_index: int) -> np.ndarray:
    """W [N, K] fp32 for one shape of a case."""
    if case.index == 0:
        return tiny_inputs()[1]
    K, N = case.shapes[shape_index]
    rng = _rng(case.index, shape_index, 0)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(case.sigma)
    return W


def activations(case: Case, shape_index: int, M: int, *, f32: bool = False) -> np.ndarray:
    """x [M, K] for one (shape, M) of a case.

    Returns fp32 for the tiny case (or when f32=True), otherwise bf16 bit
    patterns (uint16)."""
    if case.index == 0:
        x = tiny_inputs()[0]
        if M != x.shape[0]:
            raise ValueError("tiny case has M = 16")
        return x
    K, _ = case.shapes[shape_index]
    rng = _rng(case.index, shape_index, 1, M)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if case.outliers:
        k_out = max(1, int(round(0.001 * K)))
        ch = rng.choice(K, size=k_out, replace=False)
        x[:, ch] *= np.float32(20.0)
    if case.token_lognormal:
        z = rng.standard_normal((M, 1), dtype=np.float32)
        x *= np.exp(np.float32(0.5) * z).astype(np.float32)
    if f32 or case.x_dtype == "f32":
        return x
    return _to_bf16_bits(x)


def gamma_ones(K: int) -> np.ndarray:
    return np.ones((K,), np.float32)


def random_gamma(K: int, seed: int = 7) -> np.ndarray:
    """A non-trivial gain vector (used by tests to exercise gamma)."""
    rng = _rng(99, seed)
    return (np.float32(1.0) + np.float32(0.25) * rng.standard_normal((K,), dtype=np.float32)).astype(np.float32)


def outlier_channels(case: Case, shape_index: int, M: int) -> Optional[np.ndarray]:
    """The outlier channel indices used by activations() (for tests/reporting)."""
    if case.index == 0 or not case.outliers:
        return None
    K, _ = case.shapes[shape_index]
    rng = _rng(case.index, shape_index, 1, M)
    rng.standard_normal((M, K), dtype=np.float32)
    k_out = max(1, int(round(0.001 * K)))
    return np.sort(rng.choice(K, size=k_out, replace=False))


def all_problems(case: Case):
    """Yield (shape_index, K, N, M) for every problem of a case."""
    for si, (K, N) in enumerate(case.shapes):
        for M in case.ms:
            yield si, K, N, M


def group_scaled_weights(N: int, K: int, group_k: int, seed: int = 0) -> np.ndarray:
    """W [N, K] fp32 whose column groups of group_k have different spreads:
    group g ~ N(0, (0.02 * 2^u_g)^2), u_g ~ U(-1.5, 1.5) (so per-group scales
    differ by up to 8x).  PCG64(77, seed, N, K, group_k)."""
    rng = _rng(77, seed, N, K, group_k)
    u = rng.uniform(-1.5, 1.5, size=(K // group_k,)).astype(np.float32)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.repeat(np.float32(0.02) * np.exp2(u), group_k)[None, :]
    return W.astype(np.float32)


def group_scaled_activations(M: int, K: int, group_k: int, seed: int = 0) -> np.ndarray:
    """x [M, K] as bf16 bit patterns: N(0,1) with each column group scaled by
    2^v_g, v_g ~ U(-2, 2), and 0.1% x20 outlier channels.  PCG64(78, seed, M, K, group_k)."""
    rng = _rng(78, seed, M, K, group_k)
    v = rng.uniform(-2.0, 2.0, size=(K // group_k,)).astype(np.float32)
    x = rng.standard_normal((M, K), dtype=np.float32)
    x *= np.repeat(np.exp2(v), group_k)[None, :]
    ch = rng.choice(K, size=max(1, int(round(0.001 * K))), replace=False)
    x[:, ch] *= np.float32(20.0)
    return _to_bf16_bits(x)


def bitdelta_inputs(N: int, K: int, B: int, seed: int = 0):
    """BitDelta serving inputs, all bf16 bit patterns: W_base [N,K] ~ N(0, 0.02^2);
    B fine-tuned copies W_fine[b] = W_base + d, d ~ N(0, 0.002^2) (a fine-tune
    that moves each weight by about a tenth of its spread) with 5% of the
    entries left exactly equal to the base (zero deltas); one decode token
    per tenant x [B,K] ~ N(0,1).  PCG64(79, seed, N, K, B)."""
    rng = _rng(79, seed, N, K, B)
    base32 = (rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    base = _to_bf16_bits(base32)
    base_f = (base.astype(np.uint32) << 16).view(np.float32)
    fine = []
    for _ in range(B):
        d = (rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.002)).astype(np.float32)
        d[rng.random((N, K)) < 0.05] = 0.0
        f = _to_bf16_bits(base_f + d)
        fine.append(f)
    x = _to_bf16_bits(rng.standard_normal((B, K), dtype=np.float32))
    return base, fine, x


def warmup_inputs(M: int, N: int, K: int, seed: int = 0, f32: bool = False):
    """Fine-tuning inputs: W [N,K] fp32 ~ N(0, 0.02^2), x [M,K] ~ N(0,1) with
    0.1% x20 outlier channels (bf16 bits unless f32), upstream gradient
    dy [M,N] ~ N(0, 1) as bf16 bits.  PCG64(80, seed, M, N, K)."""
    rng = _rng(80, seed, M, N, K)
    W = (rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    x = rng.standard_normal((M, K), dtype=np.float32)
    ch = rng.choice(K, size=max(1, int(round(0.001 * K))), replace=False)
    x[:, ch] *= np.float32(20.0)
    dy = _to_bf16_bits(rng.standard_normal((M, N), dtype=np.float32))
    return W, (x if f32 else _to_bf16_bits(x)), dy
