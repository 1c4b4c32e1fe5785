"""Shared helpers for the GPU parity tests (inputs to the device, results back)."""
import numpy as np
import torch

import oracle
from ternary_quantized_linear_b200 import workloads


def x_to_device(x_np, device="cuda"):
    """fp32 numpy -> float32 tensor; uint16 numpy (bf16 bits) -> bfloat16 tensor."""
    if x_np.dtype == np.uint16:
        return torch.from_numpy(x_np.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x_np, np.float32)).to(device)


def bf16_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_weights(W):
    s_w, _ = oracle.weight_scale(W)
    W_p, _ = oracle.quantize_pack(W, s_w)
    return W_p, s_w


def sample_columns(N, count, seed=0):
    """Seeded column sample that always includes both ends and 128-row tile edges."""
    rng = np.random.default_rng(seed)
    must = {0, N - 1}
    for b in (31, 32, 127, 128, 255, 256):
        if b < N:
            must.add(b)
    rest = rng.choice(N, size=min(N, count), replace=False).tolist()
    return np.array(sorted(must | set(rest)), np.int64)


def case_inputs(case, shape_index, M):
    W = workloads.weights(case, shape_index)
    x = workloads.activations(case, shape_index, M)
    return x, W
