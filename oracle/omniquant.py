"""Eq. 3 -- OmniQuant's clipped MinMax quantization to a c-bit container,
with the clipping factors given (TEST INFRASTRUCTURE, like all of oracle/).

Source: "Matryoshka Quantization" explainer page, section 3.4 "Quantization
Primitives", Eq. 3 (OmniQuant's learnable quantization): the range [min, max]
of Eq. 1 becomes [beta * min(w), gamma * max(w)]:
    alpha = (gamma * max(w) - beta * min(w)) / (2^c - 1),
    z     = -(beta * min(w)) / alpha,
    q     = clamp(round(w / alpha + z), 0, 2^c - 1).
Weights outside the clipped range saturate at 0 or 2^c - 1. gamma and beta are
one pair per output channel (row), as learned by OmniQuant; learning them
needs training data and is out of scope, so they are inputs here.

The arithmetic contract is Eq. 1's (see minmax.py), with the two products
first: gmax = f32(gamma * max), bmin = f32(beta * min), d = f32(gmax - bmin),
alpha = f32(d / (2^c - 1)), z = f32(-bmin / alpha), t = f32(f32(w / alpha) + z),
q = clamp(rint_even(t), 0, 2^c - 1).

Reading where the page is silent: a row whose clipped range is empty or
inverted (alpha <= 0) gets alpha = max(|bmin| 2^-8, 2^-126) and z = -bmin / alpha,
the rule Eq. 1's constant rows follow with bmin in place of min.
"""
from __future__ import annotations

import numpy as np

from .minmax import degenerate_alpha


def _f32(a):
    """Round float64 values to the nearest float32 (ties to even), back to float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def quantize_omniquant(w: np.ndarray, gamma: np.ndarray, beta: np.ndarray, c: int = 8):
    """Quantize each row of w (N x K, float32-representable) per Eq. 3 with the
    row's clipping factors gamma[n], beta[n] (float32-representable).

    Returns (q uint8 N x K, alpha float32 N, zero float32 N).
    """
    w = np.asarray(w, dtype=np.float64)
    if w.ndim != 2:
        raise ValueError("w must be N x K")
    gamma = np.asarray(gamma, dtype=np.float64).reshape(-1)
    beta = np.asarray(beta, dtype=np.float64).reshape(-1)
    if gamma.shape[0] != w.shape[0] or beta.shape[0] != w.shape[0]:
        raise ValueError("one gamma and one beta per row")
    levels = float((1 << c) - 1)
    gmax = _f32(gamma * w.max(axis=1))
    bmin = _f32(beta * w.min(axis=1))
    alpha = _f32(_f32(gmax - bmin) / levels)
    empty = alpha <= 0.0
    alpha = np.where(empty, degenerate_alpha(bmin), alpha)
    zero = _f32(-bmin / alpha)
    with np.errstate(over="ignore", invalid="ignore"):
        t = _f32(_f32(w / alpha[:, None]) + zero[:, None])
    q = np.clip(np.rint(t), 0.0, levels)
    return q.astype(np.uint8), alpha.astype(np.float32), zero.astype(np.float32)
