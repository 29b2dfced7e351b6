"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and casts them to the storage types the
library reads (fp32, bf16 bit patterns). It holds none of the quantization,
slicing, packing or matmul arithmetic: both the CUDA path and the CPU oracle
receive the very same host arrays produced here and nothing else.

Shapes and distributions follow the Matryoshka Quantization pages' model
families (Gemma-2 2B / 9B and Mistral 7B shaped linears, FFN weights drawn
N(0, 0.02^2) or heavy-tailed Student-t(4)*0.02, activations N(0, 1)).
Every host generator is numpy.random.Generator(PCG64(seed)). The benchmark's
multi-gigabyte stack is drawn on the device instead (device_gaussian_weights,
device_activations: torch's seeded generator, the same laws), so that building
it does not take minutes of host time; a test that checks that workload draws
the same tensors again and copies the rows it samples to the host.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "gaussian_weights",
    "student_t_weights",
    "activations",
    "WORKLOADS",
    "mixnmatch_widths",
    "stack_shapes",
    "device_gaussian_weights",
    "device_activations",
]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16. NaN inputs are not expected here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + lsb) >> 16
    return rounded.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def gaussian_weights(n: int, k: int, seed: int, std: float = 0.02,
                     dtype: str = "bf16") -> np.ndarray:
    """N(0, std^2) weight matrix of n output channels by k input features.

    dtype "f32" returns float32; "bf16" returns uint16 bit patterns.
    """
    w = (_rng(seed).standard_normal((n, k), dtype=np.float64) * std).astype(np.float32)
    return w if dtype == "f32" else bf16_bits_from_f32(w)


def student_t_weights(n: int, k: int, seed: int, nu: float = 4.0, scale: float = 0.02,
                      dtype: str = "bf16") -> np.ndarray:
    """Heavy-tailed Student-t(nu) * scale weights (outliers), n x k."""
    w = (_rng(seed).standard_t(nu, size=(n, k)) * scale).astype(np.float32)
    return w if dtype == "f32" else bf16_bits_from_f32(w)


def extra_bucket_weights(n: int, k: int, seed: int, frac: float = 0.025, std: float = 0.02,
                         dtype: str = "bf16") -> np.ndarray:
    """Weights whose int8 container puts about `frac` of each row in the
    int2 extra bucket of Eq. 8 (q >= 224), as a trained Extra Precision model
    does (about 2.5%, "2.05 effective bits"): a N(0, std^2) body clipped to
    +-4 std, each row's range pinned to exactly [-4 std, 4 std], and `frac` of
    the positions drawn uniformly from [3.2 std, 4 std] (above the int2
    bucket edge at 224/255 of the range, about 3.03 std)."""
    rng = _rng(seed)
    w = np.clip(rng.standard_normal((n, k)), -4.0, 4.0)
    top = rng.random((n, k)) < frac
    w[top] = rng.uniform(3.2, 4.0, size=int(top.sum()))
    cols = rng.integers(0, k, size=(n, 2))
    cols[:, 1] = (cols[:, 0] + 1 + rng.integers(0, k - 1, size=n)) % k  # a second, distinct column
    rows = np.arange(n)
    w[rows, cols[:, 0]] = -4.0
    w[rows, cols[:, 1]] = 4.0
    w = (w * std).astype(np.float32)
    return w if dtype == "f32" else bf16_bits_from_f32(w)


def clip_factors(n: int, seed: int, lo: float = 0.6, hi: float = 1.0) -> np.ndarray:
    """Per-row clipping factors for Eq. 3 (gamma or beta): uniform in [lo, hi],
    float32. OmniQuant learns them through a sigmoid, so they lie in (0, 1);
    no training runs here, so they are drawn."""
    return _rng(seed).uniform(lo, hi, size=n).astype(np.float32)


def activations(m: int, k: int, seed: int) -> np.ndarray:
    """bf16 activations x ~ N(0, 1), m rows by k features, as uint16 bits."""
    x = _rng(seed).standard_normal((m, k), dtype=np.float64).astype(np.float32)
    return bf16_bits_from_f32(x)


# The five workloads: shapes (N x K), weight law, widths r and batch sizes M.
# Seeds: weights of the single-layer case use seed 0; the others are fixed
# per workload so every run draws identical data.
WORKLOADS = {
    "single_linear_512x1024": dict(
        mats=[("w", 512, 1024)], law="gauss", wdtype="f32", rs=[8, 4, 2], Ms=[1],
        wseed=lambda i: 0, xseed=lambda M: 1),
    "gemma2_2b_decode_layer": dict(
        mats=[("q", 2304, 2304), ("k", 2304, 2304), ("v", 2304, 2304), ("o", 2304, 2304),
              ("gate", 9216, 2304), ("up", 9216, 2304), ("down", 2304, 9216)],
        law="gauss", wdtype="bf16", rs=[4], Ms=[1, 4, 8],
        wseed=lambda i: 100 + i, xseed=lambda M: 200 + M),
    "mistral7b_mlp_heavy_tail": dict(
        mats=[("up", 14336, 4096), ("down", 4096, 14336)],
        law="student_t", wdtype="bf16", rs=[2, 4, 8], Ms=[1, 4, 16, 32],
        wseed=lambda i: 300 + i, xseed=lambda M: 400 + M),
    "mixnmatch_7b_stack": dict(
        mats=[("qkv", 6144, 4096), ("o", 4096, 4096), ("gate", 14336, 4096),
              ("up", 14336, 4096), ("down", 4096, 14336)],
        law="gauss", wdtype="bf16", rs=None, Ms=[1, 2, 4, 8, 16, 32], layers=32,
        wseed=lambda i: 1000 + i, xseed=lambda M: 2000 + M),
    "gemma2_9b_prefill": dict(
        mats=[("up", 14336, 3584), ("down", 3584, 14336)],
        law="gauss", wdtype="bf16", rs=[6, 4, 3, 2], Ms=[2048],
        wseed=lambda i: 500 + i, xseed=lambda M: 600),
}


def mixnmatch_widths(n_layers: int = 32) -> list[int]:
    """Per-layer widths of the 7B Mix'n'Match stack: int8 on the first and last
    four layers, int4 on the next four inward on each side, int2 in the middle
    (layers 8..23 of 32); the average is 4.0 bits."""
    out = []
    for l in range(n_layers):
        d = min(l, n_layers - 1 - l)
        out.append(8 if d < 4 else (4 if d < 8 else 2))
    return out


def stack_shapes(n_layers: int = 32):
    """(layer, name, N, K, weight seed) for every linear of the 7B stack."""
    mats = WORKLOADS["mixnmatch_7b_stack"]["mats"]
    res = []
    for l in range(n_layers):
        for j, (name, n, k) in enumerate(mats):
            res.append((l, name, n, k, 1000 + 5 * l + j))
    return res


def device_gaussian_weights(n: int, k: int, seed: int, device, std: float = 0.02):
    """N(0, std^2) n x k weights drawn on `device` by torch's generator seeded
    with `seed`, rounded to a bf16 tensor (the benchmark stack's weights)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return (torch.randn((n, k), generator=gen, device=device) * std).to(torch.bfloat16)


def device_activations(m: int, k: int, seed: int, device):
    """N(0, 1) activations, m x k, drawn on `device` (seeded), as a bf16 tensor."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return torch.randn((m, k), generator=gen, device=device).to(torch.bfloat16)
