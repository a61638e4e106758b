"""Pins for the e4m3 oracle (oracle/fp8.py): the value table against facts of
the format, the rounding against torch's own float8_e4m3fn conversion (an
independent implementation), ties, saturation and NaN."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8
from oracle.attention import decode_attention


def test_table_facts():
    t = fp8.E4M3_TABLE
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and math.copysign(1, t[0x80]) == -1
    assert t[0x38] == 1.0                    # exponent 7 = bias, mantissa 0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9              # smallest subnormal
    assert t[0x08] == 2.0 ** -6              # smallest normal
    assert t[0x07] == 7 * 2.0 ** -9          # largest subnormal
    nan = [c for c in range(256) if math.isnan(t[c])]
    assert nan == [0x7F, 0xFF]
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80:0xFF], -pos)
    # every finite value is an integer multiple of 2^-9 and has <= 4 significant bits
    for v in pos[1:]:
        e = math.floor(math.log2(v))
        assert (v / 2.0 ** max(e - 3, -9)).is_integer()


def test_table_matches_torch_decode():
    codes = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = fp8.E4M3_TABLE
    same = (ref == ours) | (np.isnan(ref) & np.isnan(ours))
    assert same.all()


@pytest.mark.parametrize("scale", [1.0, 0.5, 0.0173, 3.7])
def test_quantize_matches_torch(scale):
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(20000, generator=g) * 40,
                   torch.randn(20000, generator=g) * 0.01,
                   torch.rand(5000, generator=g) * 1e-3]).to(torch.float32)
    y = x / torch.tensor(scale, dtype=torch.float32)
    y = y.clamp(-448, 448)
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = fp8.quantize(x.numpy(), scale)
    assert np.array_equal(ours, ref)


def test_every_code_round_trips():
    vals = fp8.E4M3_TABLE[np.r_[0:0x7F, 0x80:0xFF]]
    codes = fp8.quantize(vals.astype(np.float32), 1.0)
    assert np.array_equal(fp8.E4M3_TABLE[codes.astype(np.int64)], vals)


def test_ties_go_to_even_mantissa():
    # 1.0625 lies half way between 1.0 (0x38) and 1.125 (0x39): even is 0x38
    # 1.1875 lies half way between 1.125 (0x39) and 1.25 (0x3A): even is 0x3A
    # 2^-10 lies half way between 0 and the smallest subnormal 2^-9: even is 0
    # 3 * 2^-10 lies between 2^-9 (0x01) and 2^-8 (0x02): even is 0x02
    x = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -1.0625, 432.0, 464.0], dtype=np.float32)
    assert list(fp8.quantize(x, 1.0)) == [0x38, 0x3A, 0x00, 0x02, 0xB8, 0x7E, 0x7E]
    # 432 is half way between 416 (0x7D) and 448 (0x7E): even mantissa is 0x7E;
    # 464 is above the largest value and saturates


def test_saturation_and_nan():
    x = np.array([449.0, 1e6, np.inf, -np.inf, -1e30, np.nan], dtype=np.float32)
    codes = fp8.quantize(x, 1.0)
    assert list(codes[:5]) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert codes[5] & 0x7F == 0x7F


def test_scale_divides_before_rounding():
    # with scale 2^k the codes are those of x * 2^-k exactly
    g = np.random.default_rng(3)
    x = (g.standard_normal(4096) * 10).astype(np.float32)
    assert np.array_equal(fp8.quantize(x, 4.0), fp8.quantize(x / 4, 1.0))
    assert np.allclose(fp8.dequantize(fp8.quantize(x, 4.0), 4.0), 4 * fp8.dequantize(fp8.quantize(x / 4, 1.0), 1.0))


def test_quantisation_error_bound():
    # relative error of a normal value is at most half a unit in the last of 3
    # mantissa bits: 2^-4
    g = np.random.default_rng(5)
    x = (g.uniform(2.0 ** -6, 448, 50000) * g.choice([-1, 1], 50000)).astype(np.float32)
    err = np.abs(fp8.dequantize(fp8.quantize(x, 1.0), 1.0) - x) / np.abs(x)
    assert err.max() <= 2.0 ** -4


def test_attention_over_dequantized_cache_closed_form():
    # one token: the output is the dequantized v0 itself; equal keys: the mean of V
    g = np.random.default_rng(9)
    D = 16
    v = (g.standard_normal((3, 1, D)) * 2).astype(np.float32)
    vq = fp8.dequantize(fp8.quantize(v, 0.05), 0.05)
    q = g.standard_normal((1, D))
    k = np.repeat(fp8.dequantize(fp8.quantize(g.standard_normal((1, 1, D)), 0.1), 0.1), 3, axis=0)
    out1 = decode_attention(q, k[:1], vq[:1], 0.25)
    assert np.allclose(out1[0], vq[0, 0], atol=0, rtol=1e-15)
    out3 = decode_attention(q, k, vq, 0.25)
    assert np.allclose(out3[0], vq[:, 0].mean(axis=0), rtol=1e-12, atol=1e-15)
