"""Exact widening of 16-bit floating-point bit patterns to float64.

Test infrastructure only (see the package docstring).

All 16-bit tensors reach the oracle as ``uint16`` arrays holding IEEE binary16
("fp16") or bfloat16 ("bf16") bit patterns, because NumPy has no bfloat16
type.  Both formats embed exactly in float64, so widening loses nothing.
"""

import numpy as np

FP16 = "fp16"
BF16 = "bf16"


def widen(bits, dtype):
    """Return the float64 values of the 16-bit patterns in ``bits``.

    fp16: reinterpret as numpy.float16, then convert (exact).
    bf16: a bfloat16 is the upper half of a float32, so shift the pattern into
    the top 16 bits of a uint32, reinterpret as float32, then convert (exact).
    """
    bits = np.asarray(bits)
    if bits.dtype != np.uint16:
        raise TypeError("expected uint16 bit patterns, got %s" % bits.dtype)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError("unknown dtype %r" % (dtype,))
