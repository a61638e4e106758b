"""Pins for the int8 oracle (oracle/int8.py): exact codes of exact multiples,
ties to even, clamping, NaN, agreement with numpy's and torch's own
round-half-to-even routines (independent implementations), the error bound of
the round trip, and attention over dequantised rows."""
import numpy as np
import torch

from oracle import int8
from oracle.attention import decode_attention


def test_exact_multiples_are_their_own_codes():
    s = 0.25                                       # a power of two: x / s is exact
    k = np.arange(-127, 128)
    assert np.array_equal(int8.quantize(k * s, s), k.astype(np.int8))
    assert np.array_equal(int8.dequantize(k.astype(np.int8), s), k * s)


def test_ties_go_to_even():
    y = np.array([0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5, 0.49999997, 0.50000006])
    assert int8.quantize(y, 1.0).tolist() == [0, 2, 2, 4, 0, -2, -2, 126, -126, 0, 1]


def test_clamp_and_nan():
    y = np.array([127.4, 127.5, 127.6, 128.0, 1e9, np.inf, -127.5, -128.0, -1e30, -np.inf, np.nan, -0.0])
    assert int8.quantize(y, 1.0).tolist() == [127, 127, 127, 127, 127, 127, -127, -127, -127, -127, 0, 0]


def test_matches_library_rounding():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200000) * 3, rng.integers(-300, 300, 20000) / 2.0]).astype(np.float32)
    s = np.float32(3.0 / 127)
    y = x / s                                      # the same fp32 division
    ref_np = np.clip(np.rint(y), -127, 127).astype(np.int8)
    ref_t = torch.clamp(torch.round(torch.from_numpy(y)), -127, 127).to(torch.int8).numpy()
    got = int8.quantize(x, float(s))
    assert np.array_equal(got, ref_np)
    assert np.array_equal(got, ref_t)


def test_round_trip_error_and_symmetry():
    rng = np.random.default_rng(4)
    s = 0.0371
    x = rng.uniform(-127 * s, 127 * s, 100000).astype(np.float32)
    err = np.abs(int8.dequantize(int8.quantize(x, s), s) - x.astype(np.float64))
    assert err.max() <= s / 2 * (1 + 1e-6)
    assert np.array_equal(int8.quantize(-x, s), -int8.quantize(x, s))


def test_attention_over_exactly_representable_rows():
    """Rows that are integer multiples of the scale survive quantisation
    unchanged, so attention over the dequantised rows is the plain attention."""
    rng = np.random.default_rng(5)
    s = 2.0 ** -5
    K = rng.integers(-127, 128, size=(50, 1, 64)) * s
    V = rng.integers(-127, 128, size=(50, 1, 64)) * s
    q = rng.standard_normal((4, 64))
    Kq = int8.dequantize(int8.quantize(K, s), s)
    Vq = int8.dequantize(int8.quantize(V, s), s)
    assert np.array_equal(Kq, K) and np.array_equal(Vq, V)
    np.testing.assert_array_equal(decode_attention(q, Kq, Vq, 0.125), decode_attention(q, K, V, 0.125))
