"""Replays an operation script on the oracle side.

Two independent stores are kept:
  * the contiguous history: each sequence's K/V rows appended in logical order,
    the "traditional" per-request layout of P1 "传统方法" and P2 §1.2 (forks copy
    the parent's rows);
  * optionally, a paged pool driven by the oracle block manager, the oracle
    scatter and the oracle block copy (P2 §3.2, §3.4).
Decode outputs come from decode_attention over either store; the tests pin
that both stores give the same rows bitwise.
"""
from __future__ import annotations

import torch

from .attention import decode_attention, split_decode_attention
from .prefix_cache import PrefixCachingModel
from . import paged


class OracleRun:
    def __init__(self, shape, num_blocks: int, free_order, keep_pool: bool = True, pool_fill=float("nan")):
        self.shape = shape
        self.bm = PrefixCachingModel(num_blocks, shape.block_size, free_order)
        self.hist = {"k": {}, "v": {}}
        dt = {"f32": torch.float32, "bf16": torch.bfloat16}[shape.dtype]
        self.pool = None
        if keep_pool:
            self.pool = {w: paged.new_pool(num_blocks, shape.num_kv_heads, shape.block_size, shape.head_dim, dt,
                                           pool_fill) for w in "kv"}
        self.records = []   # one dict per op: kind, slots, cow pairs, decode snapshot

    # -- store helpers -------------------------------------------------------
    def history(self, seq: int, which: str) -> torch.Tensor:
        chunks = self.hist[which][seq]
        if not chunks:
            return torch.empty((0, self.shape.num_kv_heads, self.shape.head_dim))
        return torch.cat(chunks) if len(chunks) > 1 else chunks[0]

    def paged_rows(self, seq: int, which: str) -> torch.Tensor:
        return paged.gather(self.pool[which], self.bm.tables[seq], self.bm.lens[seq])

    # -- replay --------------------------------------------------------------
    def apply(self, op) -> dict:
        kind = op[0]
        rec = {"kind": kind}
        if kind == "add":
            _, seq, n, src = op
            slots = self.bm.add_seq(seq, n)
            rows = {w: src(w) for w in "kv"}
            for w in "kv":
                self.hist[w][seq] = [rows[w]] if n else []
                if self.pool is not None:
                    paged.scatter(self.pool[w], rows[w], slots)
            rec.update(seq=seq, slots=slots)
        elif kind == "add_cached":
            _, seq, tokens, src = op
            slots, n_cached = self.bm.add_seq_cached(seq, tokens)
            rows = {w: src(w) for w in "kv"}
            for w in "kv":
                self.hist[w][seq] = [rows[w]] if len(tokens) else []
                if self.pool is not None:
                    paged.scatter(self.pool[w], rows[w], slots)   # -1 (cached) rows are skipped
            rec.update(seq=seq, slots=slots, n_cached=n_cached)
        elif kind == "fork":
            _, parent, child = op
            self.bm.fork(parent, child)
            for w in "kv":
                self.hist[w][child] = list(self.hist[w][parent])
            rec.update(parent=parent, child=child)
        elif kind == "append":
            _, ids, src = op
            slots, pairs = [], []
            for seq in ids:
                slot, cow = self.bm.append_slot(seq)
                slots.append(slot)
                if cow is not None:
                    pairs.append(cow)
            rows = {w: src(w) for w in "kv"}
            for w in "kv":
                for i, seq in enumerate(ids):
                    self.hist[w][seq].append(rows[w][i:i + 1])
                if self.pool is not None:
                    paged.copy_blocks(self.pool[w], pairs)   # copy before the write
                    paged.scatter(self.pool[w], rows[w], slots)
            rec.update(ids=list(ids), slots=slots, pairs=pairs)
        elif kind == "free":
            _, seq = op
            self.bm.free_seq(seq)
            for w in "kv":
                del self.hist[w][seq]
            rec.update(seq=seq)
        elif kind == "decode":
            _, ids, qsrc = op
            rec.update(ids=list(ids), tables=[self.bm.block_table(s) for s in ids],
                       lens=[self.bm.lens[s] for s in ids], qsrc=qsrc)
        else:
            raise ValueError(kind)
        self.records.append(rec)
        return rec

    def run(self, ops, upto=None):
        for op in ops[:upto]:
            self.apply(op)
        return self

    # -- outputs -------------------------------------------------------------
    def attend(self, seq: int, q_row, scale: float, use_pool: bool = False, partition_tokens: int = 0):
        """fp64 output rows [Hq][D] for one sequence with query rows q_row [Hq][D]."""
        get = self.paged_rows if use_pool else self.history
        K, V = get(seq, "k"), get(seq, "v")
        if partition_tokens:
            return split_decode_attention(q_row, K, V, scale, partition_tokens)
        return decode_attention(q_row, K, V, scale)
