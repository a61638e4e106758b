"""Oracle for prefix caching: a pool of cached prefix blocks shared across requests.

P2 §3.4 (前缀共享): the system keeps a pool of blocks holding common prefixes;
a request whose prompt starts with a cached prefix maps its first logical
blocks straight onto those physical blocks; shared blocks are counted by
reference. P3 ("技术洞察" and the outlook) adds reuse of cached system prompts
across users.

Readings (the pages give no mechanism):
  * only whole blocks of a prompt are cached; the key of prompt block i is the
    exact token sequence of blocks 0..i (so a block is reused only after the
    same full prefix), and a prompt matches block by block from block 0 until
    the first miss;
  * the cache holds its own reference on every block it lists, so a cached
    block outlives the requests that used it; a cached block that only the
    cache holds is evictable;
  * a new block comes from the front of the free list; when the free list is
    empty, the least recently released evictable block is evicted (removed
    from the cache) and used;
  * a new prompt block whose key is already listed is not listed again;
  * blocks filled by decoding are not cached.
Keys here are the exact token tuples (the C++ manager uses a hash chain with a
token check; both must make the same decisions).
"""
from __future__ import annotations

from collections import OrderedDict

from .block_manager import BlockManagerModel, NoFreeBlocks, OracleError


class PrefixCachingModel(BlockManagerModel):
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        super().__init__(num_blocks, block_size, free_order)
        self.cache: dict[tuple, int] = {}
        self.key_of: dict[int, tuple] = {}
        self.evictable: OrderedDict[int, None] = OrderedDict()   # oldest first
        self.hit_tokens = 0

    # -- allocation with eviction ----------------------------------------------
    def _available(self, exclude=()) -> int:
        return len(self.free) + sum(1 for b in self.evictable if b not in exclude)

    def _ensure_free(self) -> None:
        """If the free list is empty, evict the least recently released
        evictable block onto it."""
        if not self.free:
            if not self.evictable:
                raise NoFreeBlocks()
            b, _ = self.evictable.popitem(last=False)
            del self.cache[self.key_of.pop(b)]
            self.ref[b] = 0
            self.free.append(b)

    def _alloc(self) -> int:
        self._ensure_free()
        return self.free.popleft()

    # the base class pops the free list directly; route it through _alloc
    def add_seq(self, seq: int, num_tokens: int):
        if num_tokens < 0:
            raise OracleError("negative length")
        need = -(-num_tokens // self.block_size)
        if seq in self.tables:
            raise OracleError("sequence exists")
        if need > self._available():
            raise NoFreeBlocks()
        table = []
        for _ in range(need):
            b = self._alloc()
            self.ref[b] = 1
            table.append(b)
        self.tables[seq] = table
        self.lens[seq] = num_tokens
        return [self._slot(table, t) for t in range(num_tokens)]

    def append_slot(self, seq: int):
        if seq not in self.tables:
            from .block_manager import UnknownSeq
            raise UnknownSeq()
        t = self.lens[seq]
        needs = t % self.block_size == 0 or self.ref[self.tables[seq][t // self.block_size]] > 1
        if needs:
            self._ensure_free()
        return super().append_slot(seq)

    def add_seq_cached(self, seq: int, tokens):
        """Prefill with prefix reuse. Returns (slots, n_cached): slots of cached
        tokens are -1 (already in the pool); n_cached is a multiple of bs."""
        tokens = [int(x) for x in tokens]
        if seq in self.tables:
            raise OracleError("sequence exists")
        bs, n = self.block_size, len(tokens)
        nfull, nblocks = n // bs, -(-n // bs)
        hits = []
        for i in range(nfull):
            key = tuple(tokens[:(i + 1) * bs])
            b = self.cache.get(key)
            if b is None:
                break
            hits.append(b)
        need = nblocks - len(hits)
        if need > self._available(exclude=set(hits)):
            raise NoFreeBlocks()
        for b in hits:
            self.evictable.pop(b, None)
            self.ref[b] += 1
        table = list(hits)
        for i in range(len(hits), nblocks):
            b = self._alloc()
            self.ref[b] = 1
            table.append(b)
            if i < nfull:
                key = tuple(tokens[:(i + 1) * bs])
                if key not in self.cache:
                    self.cache[key] = b
                    self.key_of[b] = key
                    self.ref[b] += 1        # the cache's own reference
        self.tables[seq] = table
        self.lens[seq] = n
        n_cached = len(hits) * bs
        self.hit_tokens += n_cached
        slots = [-1 if t < n_cached else self._slot(table, t) for t in range(n)]
        return slots, n_cached

    def free_seq(self, seq: int) -> None:
        from .block_manager import UnknownSeq
        if seq not in self.tables:
            raise UnknownSeq()
        for b in self.tables.pop(seq):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
            elif self.ref[b] == 1 and b in self.key_of:
                self.evictable[b] = None
                self.evictable.move_to_end(b)
        del self.lens[seq]

    def prefix_stats(self) -> dict:
        return dict(cached_blocks=len(self.cache), evictable_blocks=len(self.evictable), hit_tokens=self.hit_tokens)
