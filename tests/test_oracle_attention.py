"""Pins for the oracle attention (no GPU).

Each pin is a closed form, an invariant or an independent high-precision brute
force, chosen so that a dropped term, a wrong sign, index or scale, or a
transposed operand in oracle.attention fails at least one of them.
Citation: P2 = page "PagedAttention：操作系统级 KV 缓存虚拟内存管理", §1.1
(Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V) and §4.1 (tiled softmax).
"""
import math

import mpmath
import numpy as np
import pytest

from oracle.attention import decode_attention, partition_stats, merge_partitions, split_decode_attention


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_token_returns_v0():
    q, K, V = _rand(0, 6, 16), _rand(1, 1, 3, 16), _rand(2, 1, 3, 16)
    out = decode_attention(q, K, V, 0.25)
    for h in range(6):
        assert np.array_equal(out[h], V[0, h // 2])


def test_identical_keys_give_mean_of_v():
    q = _rand(0, 4, 8)
    k = _rand(1, 1, 4, 8)
    K = np.repeat(k, 9, axis=0)
    V = _rand(2, 9, 4, 8)
    out = decode_attention(q, K, V, 0.3)
    np.testing.assert_allclose(out, V.mean(axis=0), rtol=0, atol=1e-15)


def test_zero_query_gives_mean_of_v():
    K, V = _rand(1, 7, 2, 8), _rand(2, 7, 2, 8)
    out = decode_attention(np.zeros((4, 8)), K, V, 1.0)
    np.testing.assert_allclose(out, np.repeat(V.mean(axis=0), 2, axis=0), rtol=0, atol=1e-15)


def test_two_tokens_reduce_to_logistic():
    """softmax over two scores is the logistic function of their difference."""
    q, K, V = _rand(3, 1, 5), _rand(4, 2, 1, 5), _rand(5, 2, 1, 5)
    s = 0.7
    d = s * float(sum(q[0, i] * (K[0, 0, i] - K[1, 0, i]) for i in range(5)))
    w0 = 1.0 / (1.0 + math.exp(-d))
    expect = w0 * V[0, 0] + (1.0 - w0) * V[1, 0]
    np.testing.assert_allclose(decode_attention(q, K, V, s)[0], expect, rtol=0, atol=1e-15)


def test_scale_and_exponential_base():
    """With scale 1/sqrt(d), a key whose score exceeds another's by ln 3 gets
    three times its weight: out = (v0 + 3 v1) / 4."""
    d = 64
    scale = 1.0 / math.sqrt(d)
    a = 2.0
    q = np.zeros((1, d)); q[0, 0] = a
    K = np.zeros((2, 1, d)); K[1, 0, 0] = math.log(3.0) / (scale * a)
    V = _rand(6, 2, 1, d)
    np.testing.assert_allclose(decode_attention(q, K, V, scale)[0], (V[0, 0] + 3 * V[1, 0]) / 4, rtol=0, atol=1e-14)


def test_gqa_contiguous_groups():
    """Query head h reads kv head h // G: V constant per kv head exposes the map."""
    Hq, Hkv, L, D = 8, 2, 5, 4
    q, K = _rand(7, Hq, D), _rand(8, L, Hkv, D)
    V = np.zeros((L, Hkv, D))
    for g in range(Hkv):
        V[:, g, :] = g + 1
    out = decode_attention(q, K, V, 0.5)
    for h in range(Hq):
        np.testing.assert_allclose(out[h], h // (Hq // Hkv) + 1, rtol=0, atol=1e-14)


def test_output_is_a_convex_combination_along_tokens():
    """V[t][d] = d for all t returns d: the weights sum to one along tokens, not dims."""
    L, D = 6, 8
    q, K = _rand(9, 2, D), _rand(10, L, 2, D)
    V = np.tile(np.arange(D, dtype=float), (L, 2, 1))
    np.testing.assert_allclose(decode_attention(q, K, V, 0.9), np.tile(np.arange(D), (2, 1)), rtol=0, atol=1e-14)


def test_shift_invariance():
    """Adding to every key a vector orthogonal-in-score (q . c constant) leaves the output unchanged."""
    q, K, V = _rand(11, 1, 6), _rand(12, 10, 1, 6), _rand(13, 10, 1, 6)
    c = _rand(14, 6)
    out0 = decode_attention(q, K, V, 0.4)
    out1 = decode_attention(q, K + c[None, None, :], V, 0.4)
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-13)


def test_empty_context_is_zero():
    out = decode_attention(_rand(0, 2, 4), np.zeros((0, 2, 4)), np.zeros((0, 2, 4)), 1.0)
    assert np.array_equal(out, np.zeros((2, 4)))


@pytest.mark.parametrize("seed", range(6))
def test_mpmath_brute_force(seed):
    """Element-by-element evaluation of the definition at 50 digits."""
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(1, 9)); Hkv = int(rng.integers(1, 3)); G = int(rng.integers(1, 3)); D = int(rng.integers(1, 6))
    q, K, V = rng.standard_normal((Hkv * G, D)) * 2, rng.standard_normal((L, Hkv, D)) * 2, rng.standard_normal((L, Hkv, D))
    scale = float(rng.uniform(0.1, 1.5))
    got = decode_attention(q, K, V, scale)
    mpmath.mp.dps = 50
    for h in range(Hkv * G):
        g = h // G
        scores = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(q[h, i]) * mpmath.mpf(K[t, g, i]) for i in range(D))
                  for t in range(L)]
        e = [mpmath.e ** s for s in scores]
        z = mpmath.fsum(e)
        for i in range(D):
            ref = mpmath.fsum(e[t] * mpmath.mpf(V[t, g, i]) for t in range(L)) / z
            assert abs(float(ref) - got[h, i]) <= 1e-13 * max(1.0, abs(float(ref)))


@pytest.mark.parametrize("P", [1, 2, 3, 5, 64])
def test_split_merge_equals_single_pass(P):
    q, K, V = _rand(20, 4, 16) * 3, _rand(21, 37, 2, 16), _rand(22, 37, 2, 16)
    np.testing.assert_allclose(split_decode_attention(q, K, V, 0.5, P), decode_attention(q, K, V, 0.5),
                               rtol=0, atol=1e-13)


def test_partition_stats_single_partition():
    q, K, V = _rand(23, 2, 8), _rand(24, 11, 1, 8), _rand(25, 11, 1, 8)
    m, l, o = partition_stats(q, K, V, 0.8, 0, 11)
    np.testing.assert_allclose(o / l[:, None], decode_attention(q, K, V, 0.8), rtol=0, atol=1e-15)
    x = 0.8 * (K[:, 0, :] @ q[0])
    assert m[0] == x.max()


def test_merge_weights_follow_partition_maxima():
    """Two partitions with maxima 0 and ln 2 and unit sums weight 1:2."""
    ms = np.array([[0.0], [math.log(2.0)]])
    ls = np.ones((2, 1))
    os_ = np.array([[[1.0]], [[4.0]]])
    np.testing.assert_allclose(merge_partitions(ms, ls, os_), [[(1.0 + 2 * 4.0) / 3.0]], rtol=0, atol=1e-15)
