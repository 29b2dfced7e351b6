"""CPU oracle for the Matryoshka Quantization serving path (TEST INFRASTRUCTURE).

This package is the plain, slow reference that the CUDA library is checked
against. It is test infrastructure only: nothing in the library imports it.
Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or call it.

It shares no code with the CUDA path. Everything here is float64 numpy or
Python integers, written from the Matryoshka Quantization pages:

* ``omniquant`` -- Eq. 3, OmniQuant's clipped MinMax with given per-row
                  clipping factors gamma and beta (same page, section 3.4).
* ``minmax``   -- Eq. 1, per-output-channel asymmetric MinMax int8 container
                  (page "Matryoshka Quantization" explainer, section 3.4,
                  "Quantization Primitives", Eq. 1; dequantization alpha*(q - z)).
* ``slicing``  -- Eq. 6, the MSB slicing operator S(q_c, r), and the unclamped
                  Eq. 8 variant (same page, "The Bit-Slicing Operator" and the
                  errata paragraph of section 7).
* ``planes``   -- the dense r-bit plane layout the library stores slices in
                  (the layout is this library's own; the pages fix only that
                  lower widths are stored densely as r-bit integers).
* ``chain``    -- a chained decoder stack over the sliced linears with a plain
                  stand-in glue (RMSNorm, single-token attention, SwiGLU,
                  residual), which the pages leave undefined.
* ``matmul``   -- dequantize and y = x . W_r^T in float64, the element-wise
                  tolerance bound, and the per-layer-width (Mix'n'Match) stack
                  (same page, "Mix'n'Match and Interpolative Slicing").

Parity status: every function is pinned by tests under ``tests/`` that check
it against values the pages print, closed forms, invariants or brute force.
"""
from .minmax import quantize_minmax, dequantize, FP32_CONTRACT
from .omniquant import quantize_omniquant
from .slicing import slice_code, slice_value, slice_codes, slice_table
from .planes import plane_widths, pack_rows, unpack_rows, packed_bytes, pack_rows_bigint
from .matmul import dequant_slice, linear, tolerance, stack_forward

__all__ = [
    "quantize_minmax", "dequantize", "FP32_CONTRACT", "quantize_omniquant",
    "slice_code", "slice_value", "slice_codes", "slice_table",
    "plane_widths", "pack_rows", "unpack_rows", "packed_bytes", "pack_rows_bigint",
    "dequant_slice", "linear", "tolerance", "stack_forward",
]
