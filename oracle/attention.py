"""Oracle decode attention, fp64.

The method reaches the textbook result exactly (up to rounding order): paging
only changes where K and V live, not what is computed. So the oracle is the
definition of P2 §1.1, Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V, for one
query row per head, over the gathered tokens of the sequence.

Readings (the pages are silent):
  * the scale is an argument; the workloads pass 1/sqrt(head_dim) (P2 §1.1);
  * query head h reads kv head h // G, G = Hq / Hkv (contiguous groups);
  * an empty context yields a zero output row.

`partition_stats` / `merge_partitions` state the split form: softmax over a
union of token ranges computed from per-range (max, sum of exponentials,
unnormalised weighted sum). It is the online-softmax idea of P2 §4.1 taken
across ranges instead of tiles.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def decode_attention(q, K, V, scale: float) -> np.ndarray:
    """q [Hq][D]; K, V [L][Hkv][D] (contiguous, logical order) -> out [Hq][D]."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    Hq, D = q.shape
    L, Hkv = K.shape[0], K.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of kv heads")
    G = Hq // Hkv
    out = np.zeros((Hq, D), dtype=np.float64)
    if L == 0:
        return out
    for h in range(Hq):
        g = h // G
        x = scale * (K[:, g, :] @ q[h])          # scores, [L]
        w = np.exp(x - x.max())                   # softmax numerator
        out[h] = (w @ V[:, g, :]) / w.sum()
    return out


def partition_stats(q, K, V, scale: float, start: int, stop: int):
    """For tokens [start, stop): per head (m, l, o~) with m the max score,
    l = sum exp(x - m), o~ = sum exp(x - m) v.  Natural-log domain."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    Hq, D = q.shape
    G = Hq // K.shape[1]
    m = np.empty(Hq)
    l = np.empty(Hq)
    o = np.empty((Hq, D))
    for h in range(Hq):
        g = h // G
        x = scale * (K[start:stop, g, :] @ q[h])
        m[h] = x.max()
        w = np.exp(x - m[h])
        l[h] = w.sum()
        o[h] = w @ V[start:stop, g, :]
    return m, l, o


def merge_partitions(ms, ls, os_) -> np.ndarray:
    """m = max_p m_p; l = sum_p l_p e^(m_p - m); out = sum_p o~_p e^(m_p - m) / l."""
    ms, ls, os_ = np.asarray(ms), np.asarray(ls), np.asarray(os_)   # [P][Hq], [P][Hq], [P][Hq][D]
    m = ms.max(axis=0)
    w = np.exp(ms - m)
    l = (ls * w).sum(axis=0)
    return (os_ * w[:, :, None]).sum(axis=0) / l[:, None]


def split_decode_attention(q, K, V, scale: float, partition_tokens: int) -> np.ndarray:
    """decode_attention computed partition by partition and merged."""
    L = int(K.shape[0])
    if L == 0:
        return decode_attention(q, K, V, scale)
    parts = [partition_stats(q, K, V, scale, s, min(s + partition_tokens, L))
             for s in range(0, L, partition_tokens)]
    return merge_partitions([p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts])
