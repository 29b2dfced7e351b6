"""Eq. 1 -- MinMax asymmetric quantization to a c-bit container (c = 8).

Source: "Matryoshka Quantization" explainer page, section 3.4 "Quantization
Primitives", Eq. 1:  Q(w, c) = clamp(round(w / alpha + z), 0, 2^c - 1) with
alpha = (max(w) - min(w)) / (2^c - 1) and z = -min(w) / alpha; dequantization
is alpha * (q - z). The vector w is one output channel (one row of the N x K
weight), as the pages' per-channel MinMax quantizer.

The pages write Eq. 1 in real arithmetic. The library evaluates it in IEEE
binary32 with correctly rounded single operations, so the oracle fixes the
same reading (FP32_CONTRACT below): each +, -, / is done in float64 and then
rounded to float32. For one operation on float32 operands this equals the
correctly rounded float32 result, because binary64 carries more than
2*24 + 2 significand bits (double rounding is innocuous; Figueroa, "When is
double rounding innocuous?", 1995).

Readings where the pages are silent:
* round(.) is round-half-to-even (IEEE default);
* z is kept as a real (float32), not rounded to an integer;
* a row whose alpha is 0 (max == min) gets alpha = max(|min| 2^-8, 2^-126)
  (both powers-of-two scalings, exact in float32) and z = -min / alpha
  (= -256 sign(min), or min 2^126 for |min| < 2^-118): every code is 0 and
  alpha * (0 - z) = min reproduces the row exactly. Eq. 1 divides by zero
  there; alpha on the row's own scale (rather than 1) keeps the scaled code
  sums alpha 2^(8 - r) sum_k x_k c_k of the sliced product small next to the
  row's values, as they are for every other row.
"""
from __future__ import annotations

import numpy as np

FP32_CONTRACT = (
    "d = f32(max - min); alpha = f32(d / (2^c - 1)); alpha == 0 -> alpha = max(|min| 2^-8, 2^-126); "
    "z = f32(-min / alpha); t = f32(f32(w / alpha) + z); q = clamp(rint_even(t), 0, 2^c - 1)"
)


def _f32(a):
    """Round float64 values to the nearest float32 (ties to even), back to float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def quantize_minmax(w: np.ndarray, c: int = 8):
    """Quantize each row of w (N x K, float32-representable values) per Eq. 1.

    Returns (q uint8 N x K, alpha float32 N, zero float32 N).
    """
    w = np.asarray(w, dtype=np.float64)
    if w.ndim != 2:
        raise ValueError("w must be N x K")
    levels = float((1 << c) - 1)
    mn = w.min(axis=1)
    mx = w.max(axis=1)
    d = _f32(mx - mn)
    alpha = _f32(d / levels)
    degenerate = alpha == 0.0
    alpha = np.where(degenerate, degenerate_alpha(mn), alpha)
    zero = _f32(-mn / alpha)
    with np.errstate(over="ignore", invalid="ignore"):
        t = _f32(_f32(w / alpha[:, None]) + zero[:, None])
    q = np.clip(np.rint(t), 0.0, levels)
    return q.astype(np.uint8), alpha.astype(np.float32), zero.astype(np.float32)


def degenerate_alpha(m: np.ndarray) -> np.ndarray:
    """The scale of a row with no range: max(|m| 2^-8, 2^-126), with m the
    row's minimum (Eq. 1) or clipped minimum (Eq. 3)."""
    return np.maximum(np.abs(np.asarray(m, dtype=np.float64)) * 2.0 ** -8, 2.0 ** -126)


def dequantize(q: np.ndarray, alpha: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """alpha * (q - z) in float64 (Eq. 1, "Why this form")."""
    a = np.asarray(alpha, dtype=np.float64)[:, None]
    z = np.asarray(zero, dtype=np.float64)[:, None]
    return a * (np.asarray(q, dtype=np.float64) - z)
