"""Oracle block manager: a plain Python model of the KV block pool.

Follows, step by step:
  P1 "Paged Attention 的工作原理": blocks of fixed size are handed out one at a
      time, from anywhere in the pool, when the previous block is full.
  P1 "块表（Block Table）": each request keeps an ordered list logical block i ->
      physical block.
  P2 §3.2.1: a prompt of n tokens gets ceil(n / block_size) blocks; the last may
      be partly filled.
  P2 §3.2.2 steps 2-3: before writing a new token, if the last block is full a
      new block is requested and appended to the table; the token goes to
      (block, offset).
  P2 §3.3: a finished request's blocks go back to the free pool; any free
      block may serve any request.
  P2 §3.4 and P1 "跨请求的内存共享": shared blocks carry a reference count; a
      write into a shared block first copies it, remaps the writer's table to
      the copy and drops one reference from the original (copy-on-write).

Readings where the pages are silent (shared with the C++ manager only as a
written convention, not as code):
  * the free list is a queue: allocation takes from the front, a block whose
    count reaches zero is put at the back, in the order of the freed table;
  * copy-on-write happens when the target block's count is above one;
  * every call either succeeds or leaves the state unchanged.
"""
from __future__ import annotations

from collections import deque


class OracleError(Exception):
    pass


class NoFreeBlocks(OracleError):
    pass


class UnknownSeq(OracleError):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise OracleError("bad sizes")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise OracleError("free order must be a permutation of the pool")
        self.free = deque(order)
        self.ref = [0] * self.num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- position of token t: (logical block, offset), P2 §五 --------------------
    def _slot(self, table: list[int], t: int) -> int:
        return table[t // self.block_size] * self.block_size + t % self.block_size

    def add_seq(self, seq: int, num_tokens: int) -> list[int]:
        """Prefill: ceil(n / bs) blocks from the front of the free list (P2 §3.2.1).
        Returns the slot of every prompt token, in order."""
        if seq in self.tables:
            raise OracleError("sequence exists")
        if num_tokens < 0:
            raise OracleError("negative length")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise NoFreeBlocks()
        table = [self.free.popleft() for _ in range(need)]
        for b in table:
            self.ref[b] = 1
        self.tables[seq] = table
        self.lens[seq] = num_tokens
        return [self._slot(table, t) for t in range(num_tokens)]

    def fork(self, parent: int, child: int) -> None:
        """The child's table points at the parent's blocks; every block gains a
        holder (P1 "跨请求的内存共享": both tables point at the same blocks)."""
        if parent not in self.tables:
            raise UnknownSeq()
        if child in self.tables:
            raise OracleError("sequence exists")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append_slot(self, seq: int):
        """One decode-step write position (P2 §3.2.2 steps 2-3, §3.4).
        Returns (slot, cow) where cow is (src, dst) or None."""
        if seq not in self.tables:
            raise UnknownSeq()
        table, t, bs = self.tables[seq], self.lens[seq], self.block_size
        i = t // bs
        cow = None
        if t % bs == 0:
            # the last block is full (or there is none): take a new one
            if not self.free:
                raise NoFreeBlocks()
            b = self.free.popleft()
            self.ref[b] = 1
            table.append(b)
        else:
            src = table[i]
            if self.ref[src] > 1:
                # shared, read-only block: copy before writing
                if not self.free:
                    raise NoFreeBlocks()
                dst = self.free.popleft()
                self.ref[src] -= 1
                self.ref[dst] = 1
                table[i] = dst
                cow = (src, dst)
        self.lens[seq] = t + 1
        return self._slot(table, t), cow

    def free_seq(self, seq: int) -> None:
        """Release a finished request (P2 §3.3)."""
        if seq not in self.tables:
            raise UnknownSeq()
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    # -- observation ---------------------------------------------------------
    def block_table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def stats(self) -> dict:
        """Slots in allocated blocks vs slots holding a token (P1
        "内存浪费的两种形式": reserved but unused space is internal waste)."""
        fill: dict[int, int] = {}
        for seq, table in self.tables.items():
            L = self.lens[seq]
            for i, b in enumerate(table):
                n = min(self.block_size, L - i * self.block_size)
                fill[b] = max(fill.get(b, 0), n)
        allocated = (self.num_blocks - len(self.free)) * self.block_size
        used = sum(fill.values())
        return dict(free_blocks=len(self.free), used_slots=used, allocated_slots=allocated,
                    internal_waste=allocated - used)


def contiguous_waste(lengths, max_len: int) -> int:
    """Slots left empty when every request reserves max_len contiguous slots
    (the "traditional" method of P1 "传统方法" and P2 §1.2)."""
    return sum(max_len - int(n) for n in lengths)
