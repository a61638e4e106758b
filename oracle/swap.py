"""Oracle for swapping sequences' blocks between GPU and host memory.

P2 §五 (页面置换): when GPU memory runs short, inactive blocks can be moved out
to CPU memory, like an OS paging out; P2 §八 lists a GPU / CPU / NVMe hierarchy
as the direction this takes.

Readings (the pages give no mechanism):
  * the unit is a whole sequence: swap-out moves every block of its table to
    host blocks and releases the device blocks (one reference each: a block
    shared with a live sequence stays on the device for the other holder);
    swap-in brings them back into fresh device blocks;
  * host blocks come from their own FIFO free list (front = next, back = most
    recently freed), exactly like the device list;
  * a swapped-out sequence keeps its length; it cannot append or decode until
    it is swapped in; the emitted pairs are (device block, host block) in table
    order for swap-out and (host block, device block) for swap-in, and the copy
    must run on the stream before anything reuses the released blocks;
  * every call is all or nothing.
"""
from __future__ import annotations

from collections import deque

from .block_manager import NoFreeBlocks, OracleError, UnknownSeq
from .prefix_cache import PrefixCachingModel


class SwappingModel(PrefixCachingModel):
    def __init__(self, num_blocks: int, block_size: int, free_order=None, host_blocks: int = 0):
        super().__init__(num_blocks, block_size, free_order)
        self.host_free = deque(range(host_blocks))
        self.swapped: dict[int, tuple[list[int], int]] = {}   # seq -> (host table, length)

    def swap_out(self, seq: int):
        if seq not in self.tables:
            raise UnknownSeq()
        table = self.tables[seq]
        if len(table) > len(self.host_free):
            raise NoFreeBlocks()
        host = [self.host_free.popleft() for _ in table]
        pairs = list(zip(table, host))
        L = self.lens[seq]
        self.free_seq(seq)                 # releases one reference per device block
        self.swapped[seq] = (host, L)
        return pairs

    def swap_in(self, seq: int):
        if seq not in self.swapped:
            raise UnknownSeq()
        host, L = self.swapped[seq]
        if len(host) > self._available():
            raise NoFreeBlocks()
        dev = []
        for _ in host:
            b = self._alloc()
            self.ref[b] = 1
            dev.append(b)
        del self.swapped[seq]
        self.tables[seq] = dev
        self.lens[seq] = L
        for h in host:
            self.host_free.append(h)
        return list(zip(host, dev))

    def add_seq(self, seq, num_tokens):
        if seq in self.swapped:
            raise OracleError("sequence exists")
        return super().add_seq(seq, num_tokens)

    def free_seq(self, seq: int) -> None:
        if seq in self.swapped:
            host, _ = self.swapped.pop(seq)
            for h in host:
                self.host_free.append(h)
            return
        super().free_seq(seq)


def swap_copy(dev_pool, host_pool, pairs, out: bool) -> None:
    """Bit copy of whole blocks: device -> host for swap-out, host -> device for swap-in."""
    for a, b in pairs:
        if out:
            host_pool[int(b)] = dev_pool[int(a)].clone()
        else:
            dev_pool[int(b)] = host_pool[int(a)].clone()
