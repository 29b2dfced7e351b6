"""Dequantized sliced weights, y = x . W_r^T, the tolerance bound, and the
per-layer-width stack.

Sources on the "Matryoshka Quantization" explainer page:
* dequantization alpha * (q - z) (section 3.4, Eq. 1, "Why this form");
* the sliced model uses S(q, r) in place of q (Eq. 6; section 3.2 "at
  deployment ... lower-precision models are extracted on-the-fly by slicing");
* Mix'n'Match: each layer may use its own width (section "Mix'n'Match and
  Interpolative Slicing"; "Reverse Pyramid" puts int8 at the edges and int2
  in the middle).

Everything is float64: x is the exact value of its bf16 input, alpha and z are
their float32 values, and W_r[n, k] = alpha_n * (S(q[n, k], r) - z_n).
"""
from __future__ import annotations

import numpy as np

from .minmax import quantize_minmax
from .slicing import slice_codes


def dequant_slice(q: np.ndarray, alpha: np.ndarray, zero: np.ndarray, r: int,
                  c: int = 8, clamp: bool = True) -> np.ndarray:
    """W_r = alpha * (S(q, r) - z) in float64, N x K (S from Eq. 6, or from
    the unclamped Eq. 8 when clamp=False)."""
    s_val = slice_codes(q, r, c, clamp).astype(np.float64) * float(1 << (c - r))
    a = np.asarray(alpha, dtype=np.float64)[:, None]
    z = np.asarray(zero, dtype=np.float64)[:, None]
    return a * (s_val - z)


def linear(x: np.ndarray, w_r: np.ndarray) -> np.ndarray:
    """y = x . W_r^T in float64 (M x K times (N x K)^T -> M x N)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w_r, dtype=np.float64).T


def tolerance(x: np.ndarray, w_r: np.ndarray, rel: float = 1e-3, abs_: float = 1e-6) -> np.ndarray:
    """Per-element bound rel * sum_k |x[m,k]| |W_r[n,k]| + abs_ (M x N)."""
    return rel * (np.abs(np.asarray(x, dtype=np.float64)) @ np.abs(w_r).T) + abs_


def stack_forward(linears, widths, layer_of_lin, xs):
    """Mix'n'Match stack: linear i uses width widths[layer_of_lin[i]].

    linears: list of (w N x K float values, x index); xs: list of M x K float64.
    Each weight is quantized per Eq. 1, sliced per Eq. 6 at its layer's width
    and applied to its input. Returns the list of M x N outputs.
    """
    outs = []
    for i, (w, xi) in enumerate(linears):
        q, a, z = quantize_minmax(w)
        w_r = dequant_slice(q, a, z, widths[layer_of_lin[i]])
        outs.append(linear(xs[xi], w_r))
    return outs
