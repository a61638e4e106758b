"""Oracle for paged prefill attention (causal, over the block table).

P2 §3.2.1 (预填充阶段): the prompt is fed in at once; its K, V are computed and
written into the sequence's blocks. The attention of those prompt tokens is the
same softmax(q K^T / sqrt(d)) V of P2 §1.1, each token seeing every earlier
token of its sequence and itself (autoregressive order, P1 "KV Cache 快速回顾":
a token attends to the tokens before it).

Reading: a call may carry only the last n tokens of a sequence of length L
(chunked prefill): new token i sits at position L - n + i and sees positions
0 .. L - n + i, the earlier ones already in the cache.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64, decode_attention


def prefill_attention(q_rows, K, V, scale: float) -> np.ndarray:
    """q_rows [n][Hq][D]; K, V [L][Hkv][D] (logical order, n <= L) -> out [n][Hq][D]."""
    q_rows = _f64(q_rows)
    n, L = q_rows.shape[0], int(K.shape[0])
    if n > L:
        raise ValueError("more new tokens than context")
    out = np.empty(q_rows.shape)
    for i in range(n):
        pos = L - n + i
        out[i] = decode_attention(q_rows[i], K[:pos + 1], V[:pos + 1], scale)
    return out


def prefill_attention_masked(q_rows, K, V, scale: float) -> np.ndarray:
    """The same attention written as one masked matrix softmax per head (an
    independent formulation used to pin prefill_attention)."""
    q, K, V = _f64(q_rows), _f64(K), _f64(V)
    n, Hq, D = q.shape
    L, Hkv = K.shape[0], K.shape[1]
    G = Hq // Hkv
    pos = np.arange(L - n, L)                      # position of each new token
    mask = np.arange(L)[None, :] <= pos[:, None]   # [n][L]
    out = np.empty((n, Hq, D))
    for h in range(Hq):
        S = scale * q[:, h, :] @ K[:, h // G, :].T
        S = np.where(mask, S, -np.inf)
        S -= S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ V[:, h // G, :]
    return out
