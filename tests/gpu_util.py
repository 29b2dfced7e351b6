"""Helpers for the GPU tests: host <-> device transfers and the oracle-side
expected values. Inputs always come from synth/ or the oracle, never from the
CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth

DEV = "cuda:0"


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(DEV)


def empty_u8(n: int) -> torch.Tensor:
    # allocation rounded to 16 bytes keeps every buffer 16-byte aligned
    return torch.empty(max(n, 16), dtype=torch.uint8, device=DEV)


def weights(law: str, n: int, k: int, seed: int, dtype: str = "bf16"):
    """Returns (host bits or floats as stored, float64 values)."""
    if law == "gauss":
        w = synth.gaussian_weights(n, k, seed, dtype=dtype)
    else:
        w = synth.student_t_weights(n, k, seed, dtype=dtype)
    vals = synth.f32_from_bf16_bits(w) if dtype == "bf16" else w
    return w, vals.astype(np.float64)


def gpu_quantize(w_host: np.ndarray, dtype: str):
    n, k = w_host.shape
    w_d = to_dev(w_host)
    q = torch.empty((n, k), dtype=torch.uint8, device=DEV)
    a = torch.empty(n, dtype=torch.float32, device=DEV)
    z = torch.empty(n, dtype=torch.float32, device=DEV)
    mq.quantize_int8(w_d, mq.MQ_F32 if dtype == "f32" else mq.MQ_BF16, n, k, q, a, z)
    torch.cuda.synchronize()
    return q, a, z


def gpu_pack(q_dev: torch.Tensor, r: int) -> torch.Tensor:
    n, k = q_dev.shape
    packed = empty_u8(mq.packed_bytes(n, k, r))
    mq.slice_pack(q_dev, n, k, r, packed)
    return packed


def gpu_linear(x_bits: np.ndarray, packed, a_dev, z_dev, n: int, r: int) -> np.ndarray:
    m, k = x_bits.shape
    x_d = to_dev(x_bits)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear(x_d, m, k, packed, a_dev, z_dev, n, r, y)
    mq.device_status()
    return y.cpu().numpy().astype(np.float64)


def check_linear(y_gpu: np.ndarray, x_vals: np.ndarray, w_r: np.ndarray, label: str = ""):
    """Element-wise: |y_gpu - y_ref| <= 1e-3 sum|x||W_r| + 1e-6 (the stated tolerance)."""
    y_ref = oracle.linear(x_vals, w_r)
    tol = oracle.tolerance(x_vals, w_r)
    assert np.all(np.isfinite(y_gpu)), f"{label}: non-finite output (unwritten element?)"
    err = np.abs(y_gpu - y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{label}: {bad.sum()} of {bad.size} outside tolerance; first {tuple(i)}: "
            f"gpu {y_gpu[tuple(i)]!r} ref {y_ref[tuple(i)]!r} tol {tol[tuple(i)]!r}")
    return float((err / tol).max())
