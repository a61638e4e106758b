"""Pins for the oracle prefix cache (no GPU).

P2 = page "PagedAttention：操作系统级 KV 缓存虚拟内存管理", §3.4 (a pool of common-prefix
blocks; a request hitting a prefix maps its first logical blocks onto the shared
physical blocks; shared blocks are counted by reference). P3 = page
"PagedAttention 和 vLLM" (cached system prompts reused across requests).
"""
import pytest

from oracle.block_manager import NoFreeBlocks
from oracle.prefix_cache import PrefixCachingModel


def _check(m):
    counts = [0] * m.num_blocks
    for t in m.tables.values():
        for b in t:
            counts[b] += 1
    for b in m.key_of:
        counts[b] += 1                     # the cache's own reference
    assert counts == m.ref
    free = set(m.free)
    assert len(free) == len(m.free)
    assert free.isdisjoint(m.key_of)       # a listed block is never on the free list
    for b in m.evictable:
        assert b in m.key_of and m.ref[b] == 1
    held = {b for b in range(m.num_blocks) if m.ref[b] > 0}
    assert held | free == set(range(m.num_blocks)) and held.isdisjoint(free)
    for key, b in m.cache.items():
        assert m.key_of[b] == key and len(key) % m.block_size == 0


def test_shared_prefix_maps_to_the_same_blocks():
    """P2 §3.4: the second request's first blocks are the first request's blocks."""
    m = PrefixCachingModel(16, 4, list(range(16)))
    a = [1, 2, 3, 4, 5, 6, 7, 8, 9, 10]
    s1, c1 = m.add_seq_cached(1, a)
    s2, c2 = m.add_seq_cached(2, a[:8] + [50, 51, 52])
    assert c1 == 0 and c2 == 8
    assert m.block_table(2)[:2] == m.block_table(1)[:2]
    assert m.block_table(2)[2] != m.block_table(1)[2]        # the partial block is never shared
    assert s2[:8] == [-1] * 8 and s2[8] == m.block_table(2)[2] * 4
    assert m.ref[m.block_table(1)[0]] == 3                   # two requests + the cache
    _check(m)


def test_key_is_the_whole_prefix():
    """The same 4 tokens after a different prefix are a different block."""
    m = PrefixCachingModel(16, 4, list(range(16)))
    m.add_seq_cached(1, [1, 2, 3, 4, 9, 9, 9, 9])
    _, c = m.add_seq_cached(2, [7, 7, 7, 7, 9, 9, 9, 9])
    assert c == 0
    _, c = m.add_seq_cached(3, [1, 2, 3, 4, 9, 9, 9, 9, 0])
    assert c == 8
    _check(m)


def test_cache_outlives_requests_and_evicts_lru():
    m = PrefixCachingModel(6, 2, list(range(6)))
    m.add_seq_cached(1, [1, 1, 2, 2])       # blocks 0, 1 listed
    m.add_seq_cached(2, [3, 3])             # block 2 listed
    m.free_seq(1)                           # 0, 1 evictable (in table order)
    m.free_seq(2)                           # then 2
    assert list(m.evictable) == [0, 1, 2] and list(m.free) == [3, 4, 5]
    _, c = m.add_seq_cached(3, [1, 1, 2, 2, 5])   # hits 0, 1; 5 -> block 3
    assert c == 4 and list(m.evictable) == [2]
    m.add_seq_cached(4, [8, 8, 8, 8, 8, 8])       # needs 3: 4, 5, then evicts 2
    assert m.block_table(4) == [4, 5, 2]
    assert (3, 3) not in m.cache and m.prefix_stats()["evictable_blocks"] == 0
    with pytest.raises(NoFreeBlocks):
        m.add_seq_cached(5, [9, 9])
    _check(m)


def test_uncached_prefill_and_appends_evict_too():
    m = PrefixCachingModel(3, 2, [0, 1, 2])
    m.add_seq_cached(1, [1, 1, 2, 2])
    m.free_seq(1)
    m.add_seq(2, 1)                   # block 2 from the free list
    slot, cow = m.append_slot(2)      # fills block 2
    m.append_slot(2)                  # needs a block: evicts 0 (oldest)
    assert m.block_table(2) == [2, 0] and list(m.evictable) == [1]
    _check(m)


def test_exhaustion_leaves_state_unchanged():
    m = PrefixCachingModel(4, 2, [0, 1, 2, 3])
    m.add_seq_cached(1, [1, 1, 2, 2, 3])
    snap = (list(m.free), list(m.ref), dict(m.cache), list(m.evictable))
    with pytest.raises(NoFreeBlocks):
        m.add_seq_cached(2, [9, 9, 9, 9])
    assert snap == (list(m.free), list(m.ref), dict(m.cache), list(m.evictable))
