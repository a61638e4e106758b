"""Pins for the oracle prefill attention (no GPU). P2 = page "PagedAttention：操作系统级
KV 缓存虚拟内存管理", §1.1 (the attention formula) and §3.2.1 (prefill)."""
import numpy as np
import pytest

from oracle.attention import decode_attention
from oracle.prefill import prefill_attention, prefill_attention_masked


def _r(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("n,L,G", [(1, 1, 1), (5, 5, 2), (7, 20, 4), (16, 16, 8), (3, 40, 1)])
def test_loop_equals_masked_matrix_form(n, L, G):
    hkv = 2
    q, K, V = _r(n, n, hkv * G, 8) * 2, _r(L, L, hkv, 8), _r(L + 1, L, hkv, 8)
    np.testing.assert_allclose(prefill_attention(q, K, V, 0.3), prefill_attention_masked(q, K, V, 0.3),
                               rtol=0, atol=1e-13)


def test_first_prompt_token_returns_v0():
    q, K, V = _r(1, 4, 2, 8), _r(2, 4, 1, 8), _r(3, 4, 1, 8)
    out = prefill_attention(q, K, V, 1.0)
    assert np.array_equal(out[0, 0], V[0, 0]) and np.array_equal(out[0, 1], V[0, 0])


def test_last_token_is_decode():
    """The last new token sees the whole context: it is the decode step."""
    q, K, V = _r(4, 6, 4, 8), _r(5, 30, 2, 8), _r(6, 30, 2, 8)
    np.testing.assert_array_equal(prefill_attention(q, K, V, 0.5)[-1], decode_attention(q[-1], K, V, 0.5))


def test_chunked_equals_whole():
    """Prefill in two chunks (the second seeing the first through the cache)
    equals one prefill of the whole prompt."""
    q, K, V = _r(7, 24, 2, 8), _r(8, 24, 1, 8), _r(9, 24, 1, 8)
    whole = prefill_attention(q, K, V, 0.4)
    first = prefill_attention(q[:10], K[:10], V[:10], 0.4)
    second = prefill_attention(q[10:], K, V, 0.4)
    np.testing.assert_allclose(np.concatenate([first, second]), whole, rtol=0, atol=1e-14)


def test_causality():
    """Changing a later key/value does not change earlier outputs."""
    q, K, V = _r(10, 12, 2, 8), _r(11, 12, 2, 8), _r(12, 12, 2, 8)
    a = prefill_attention(q, K, V, 0.7)
    K2, V2 = K.copy(), V.copy()
    K2[8:] += 5.0
    V2[8:] -= 3.0
    b = prefill_attention(q, K2, V2, 0.7)
    np.testing.assert_array_equal(a[:8], b[:8])
    assert not np.allclose(a[8:], b[8:])
