"""Eq. 6 -- the MSB slicing operator S(q_c, r), and the unclamped Eq. 8.

Source: "Matryoshka Quantization" explainer page, "The Bit-Slicing Operator"
(Eq. 6):  S(q_c, r) = clamp(round(q_c / 2^(c-r)), 0, 2^r - 1) * 2^(c-r).
The same paragraph fixes the rounding: the first dropped bit (the (r+1)-th
MSB) decides, 1 rounds up and 0 rounds down -- i.e. round half up on
q_c / 2^(c-r). Its worked example maps 53 to 64 at r = 2. The errata
paragraph (section 7) gives the earlier, unclamped form (Eq. 8), which lets
the top bucket reach 2^r (the "Extra Precision" variant).

The "code" is the r-bit integer clamp(round(q / 2^(c-r)), 0, 2^r - 1); the
"value" is code * 2^(c-r), which lives on the c-bit scale.
"""
from __future__ import annotations

import numpy as np


def slice_code(q: int, r: int, c: int = 8, clamp: bool = True) -> int:
    """r-bit code of one c-bit integer q (Eq. 6; Eq. 8 when clamp=False)."""
    q = int(q)
    if not (0 <= q < (1 << c)):
        raise ValueError("q out of range")
    if not (1 <= r <= c):
        raise ValueError("r out of range")
    step = 1 << (c - r)                      # 2^(c-r)
    # round(q / step), ties upward: floor(q/step + 1/2) = floor((2q + step) / (2 step))
    rounded = (2 * q + step) // (2 * step)
    if clamp:
        rounded = min(max(rounded, 0), (1 << r) - 1)
    return rounded


def slice_value(q: int, r: int, c: int = 8, clamp: bool = True) -> int:
    """S(q, r) on the c-bit scale: code * 2^(c-r)."""
    return slice_code(q, r, c, clamp) * (1 << (c - r))


def slice_table(r: int, c: int = 8, clamp: bool = True) -> np.ndarray:
    """Codes of all 2^c container values (brute-force table, one entry per q)."""
    return np.array([slice_code(q, r, c, clamp) for q in range(1 << c)], dtype=np.int64)


def slice_codes(q: np.ndarray, r: int, c: int = 8, clamp: bool = True) -> np.ndarray:
    """Codes of a whole uint8 array, by lookup in the brute-force table."""
    return slice_table(r, c, clamp)[np.asarray(q, dtype=np.int64)]
