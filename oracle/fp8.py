"""Oracle for an 8-bit (e4m3) KV cache.  TEST INFRASTRUCTURE ONLY.

P3 ("PagedAttention 和 vLLM", the section on its future) expects paged KV
management to be combined with quantisation. The pages fix no format; the
reading taken here is the common one for KV caches:

  * element format e4m3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent 0 is subnormal; the all-ones exponent is an ordinary binade
    except for mantissa 111, which is NaN; no infinities, largest finite 448);
  * one positive scale per tensor (k_scale for K, v_scale for V): a stored code
    c stands for value(c) * scale;
  * quantisation divides in fp32 (x / scale, correctly rounded), then takes the
    nearest e4m3 value, ties to the code with an even mantissa; finite values
    beyond +-448 and infinities become +-448 (saturation), NaN stays NaN;
  * the attention reads value(c) * scale; everything after is the plain
    attention of oracle.attention.

The value table is built from the bit layout above, and the rounding is a
nearest-neighbour search over that table, so that nothing here relies on a
library's fp8 converter (the tests compare against one).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of an 8-bit code (NaN for the two NaN codes)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)

# finite non-negative codes in increasing value order: 0x00 .. 0x7E
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = E4M3_TABLE[:0x7F]


def _nearest_nonneg(y: np.ndarray) -> np.ndarray:
    """Code of the nearest value to each y in [0, 448], ties to even mantissa."""
    hi = np.searchsorted(_POS_VALUES, y, side="left")   # first value >= y
    hi = np.clip(hi, 0, len(_POS_VALUES) - 1)
    lo = np.clip(hi - 1, 0, None)
    d_lo = y - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - y
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((_POS_CODES[hi] & 1) == 0))
    code = np.where(take_hi, _POS_CODES[hi], _POS_CODES[lo])
    return np.where(_POS_VALUES[hi] == y, _POS_CODES[hi], code)


def quantize(x, scale: float) -> np.ndarray:
    """Codes (uint8) of x / scale; x is any real array (read as fp32)."""
    x = np.asarray(x, dtype=np.float32)
    y = (x / np.float32(scale)).astype(np.float32)           # fp32 division
    nan = np.isnan(y)
    a = np.minimum(np.abs(np.where(nan, 0, y)).astype(np.float64), E4M3_MAX)
    code = _nearest_nonneg(a)
    code = np.where(np.signbit(y), code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def dequantize(codes, scale: float) -> np.ndarray:
    """value(code) * scale in fp64."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8).astype(np.int64)] * float(scale)
