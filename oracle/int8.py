"""Oracle for an 8-bit integer (int8) KV cache.  TEST INFRASTRUCTURE ONLY.

P3 ("PagedAttention 和 vLLM", the section on its future) expects paged KV
management to be combined with quantisation; the pages fix no format. The
integer reading taken here is the symmetric per-tensor one:

  * one positive scale per tensor (k_scale for K, v_scale for V): a stored
    code c, an integer in [-127, 127], stands for c * scale (-128 is never
    written, so negation maps codes onto codes);
  * quantisation divides in fp32 (x / scale, correctly rounded), takes the
    nearest integer, ties to the even one, and clamps to [-127, 127] (so
    infinities become +-127); NaN has no integer code and becomes 0;
  * the attention reads c * scale; everything after is the plain attention
    of oracle.attention.

The rounding is written out (floor, then a comparison of the fraction with
one half) so that the tests can hold it against library rounding routines.
"""
from __future__ import annotations

import numpy as np

INT8_MAX = 127


def quantize(x, scale: float) -> np.ndarray:
    """Codes (int8) of x / scale; x is any real array (read as fp32)."""
    x = np.asarray(x, dtype=np.float32)
    y = (x / np.float32(scale)).astype(np.float32)           # fp32 division
    y = np.where(np.isnan(y), 0.0, y).astype(np.float64)
    y = np.clip(y, -INT8_MAX, INT8_MAX)
    f = np.floor(y)
    frac = y - f                                             # exact in fp64
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(f, 2.0) == 1.0))
    return (f + up).astype(np.int8)


def dequantize(codes, scale: float) -> np.ndarray:
    """code * scale in fp64."""
    return np.asarray(codes, dtype=np.int8).astype(np.float64) * float(scale)
