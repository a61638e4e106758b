"""CPU pins of the exact-widening identities the 8-bit kernels rely on (no GPU):
an int8 code c, biased by 128 and placed as the low byte under the exponent
of 1024 (f16) or 2^23 (fp32), reads back as 1024 + c + 128 or 2^23 + c + 128,
so one subtraction recovers c exactly; every e4m3 value is exact in f16. The
kernels' byte permutes and conversions implement these identities; the GPU
parity tests check the kernels themselves."""
import numpy as np
import torch

from oracle import fp8
from paged_kv_cache_361_b200 import PagedKVCache


def test_int8_to_f16_by_bias_and_exponent():
    c = np.arange(-128, 128)
    u = (c.astype(np.int64) ^ 0x80) & 0xFF            # sign bit flipped: c + 128 as an unsigned byte
    assert np.array_equal(u, c + 128)
    h = (0x6400 | u).astype(np.uint16).view(np.float16)
    assert np.array_equal(h.astype(np.float64), 1024.0 + c + 128)
    diff = (h - np.float16(1152.0)).astype(np.float16)  # one f16 subtraction, exact
    assert np.array_equal(diff.astype(np.float64), c.astype(np.float64))


def test_int8_to_fp32_by_bias_and_exponent():
    c = np.arange(-128, 128)
    u = (c.astype(np.int64) ^ 0x80) & 0xFF
    f = (0x4B000000 | u).astype(np.uint32).view(np.float32)
    assert np.array_equal((f - np.float32(8388736.0)).astype(np.float64), c.astype(np.float64))


def test_e4m3_values_are_exact_in_f16():
    finite = ~np.isnan(fp8.E4M3_TABLE)
    v = fp8.E4M3_TABLE[finite]
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)


def test_int8_pool_fill_uses_the_unwritten_code():
    """A NaN fill of an int8 pool stores -128, a code quantisation never writes."""
    cache = PagedKVCache(4, 1, 16, 64, torch.int8, "cpu", fill=float("nan"), k_scale=0.1, v_scale=0.1)
    assert int(cache.k_cache.min()) == -128 and int(cache.k_cache.max()) == -128
    assert torch.equal(cache.k_cache, cache.v_cache)
