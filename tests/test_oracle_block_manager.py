"""Pins for the oracle block manager (no GPU).

Citations: P1 = page "Paged Attention：大模型推理显存优化的核心方案", P2 = page
"PagedAttention：操作系统级 KV 缓存虚拟内存管理".
"""
import copy
import json
import os

import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, NoFreeBlocks, UnknownSeq, OracleError, contiguous_waste
from paged_kv_cache_361_b200 import workloads as W


def _p1(golden_dir):
    with open(os.path.join(golden_dir, "p1_worked_example.json")) as f:
        return json.load(f)


def _free_order_starting(first, n):
    rest = [b for b in range(n) if b not in first]
    return list(first) + rest


def _check_blocks(g, bm, seq):
    bs = g["block_size"]
    table = bm.block_table(seq)
    assert table == g["block_table"]
    # token i of the example sits in block table[i // bs] at offset i % bs
    for i, tok in enumerate(g["tokens"]):
        blk, off = divmod(i, bs)
        assert g["blocks"][blk][off] == tok
    st = bm.stats()
    assert st["internal_waste"] == g["last_block_empty_slots"]
    assert st["allocated_slots"] - st["used_slots"] == g["last_block_empty_slots"]


def test_p1_worked_example_prefill(golden_dir):
    """P1 "Paged Attention 的工作原理" / "块表": 10 tokens, blocks of 4 -> 3 blocks
    at the table's physical positions, 2 empty slots in the last."""
    g = _p1(golden_dir)
    bm = BlockManagerModel(16, g["block_size"], _free_order_starting(g["block_table"], 16))
    slots = bm.add_seq(0, len(g["tokens"]))
    table = g["block_table"]
    assert slots == [table[i // 4] * 4 + i % 4 for i in range(10)]
    assert slots == [20, 21, 22, 23, 48, 49, 50, 51, 12, 13]
    _check_blocks(g, bm, 0)


def test_p1_worked_example_incremental(golden_dir):
    """P1's walk-through allocates a block only when the previous one is full."""
    g = _p1(golden_dir)
    bm = BlockManagerModel(16, g["block_size"], _free_order_starting(g["block_table"], 16))
    bm.add_seq(0, 0)
    allocated_at = []
    for t in range(len(g["tokens"])):
        before = len(bm.block_table(0))
        slot, cow = bm.append_slot(0)
        assert cow is None
        if len(bm.block_table(0)) != before:
            allocated_at.append(t)
    assert allocated_at == [0, 4, 8]   # blocks 1, 2, 3 of the walk-through
    _check_blocks(g, bm, 0)


def test_p1_contiguous_waste(golden_dir):
    """P1 "传统方法": 16 reserved slots for 10 tokens leave 6 empty."""
    g = _p1(golden_dir)
    assert contiguous_waste([len(g["tokens"])], g["contiguous_reserved_slots"]) == g["contiguous_wasted_slots"]


def _invariants(bm):
    # every reference is counted exactly once
    counts = [0] * bm.num_blocks
    for table in bm.tables.values():
        for b in table:
            counts[b] += 1
    assert counts == bm.ref
    used = {b for b in range(bm.num_blocks) if bm.ref[b] > 0}
    free = list(bm.free)
    assert len(free) == len(set(free))
    assert used.isdisjoint(free)
    assert used | set(free) == set(range(bm.num_blocks))
    # waste only in the last block of each sequence (P1 "为什么 Paged Attention 如此高效", P2 §3.3)
    for seq, table in bm.tables.items():
        L = bm.lens[seq]
        assert len(table) == -(-L // bm.block_size)
        for i in range(len(table) - 1):
            assert L - i * bm.block_size >= bm.block_size


def test_invariants_through_batching_trace():
    tr = W.continuous_batching(seed=3, num_live=24, steps=60, num_blocks=4000, p_finish=0.05)
    ops = W.batching_ops(tr)
    bm = BlockManagerModel(tr.num_blocks, tr.shape.block_size, tr.free_order)
    n_free = 0
    for op in ops:
        if op[0] == "add":
            bm.add_seq(op[1], op[2])
        elif op[0] == "append":
            for s in op[1]:
                bm.append_slot(s)
        elif op[0] == "free":
            bm.free_seq(op[1])
            n_free += 1
        _invariants(bm)
    assert n_free > 0


def test_freed_blocks_go_to_back_and_are_reused():
    """P2 §3.3: freed blocks return to the pool and any request may take them."""
    bm = BlockManagerModel(6, 2, [0, 1, 2, 3, 4, 5])
    bm.add_seq(10, 4)          # blocks 0, 1
    bm.add_seq(11, 2)          # block 2
    bm.free_seq(10)            # free list: 3, 4, 5, 0, 1
    assert list(bm.free) == [3, 4, 5, 0, 1]
    bm.add_seq(12, 8)          # 3, 4, 5, 0
    assert bm.block_table(12) == [3, 4, 5, 0]
    _invariants(bm)


def test_copy_on_write_parallel_sampling():
    """P2 §3.4: the first write into a shared partial block copies it; the last
    holder writes in place; full shared blocks are never copied."""
    bm = BlockManagerModel(64, 4, list(range(64)))
    bm.add_seq(0, 10)                      # blocks 0, 1, 2 (2 holds 2 tokens)
    for j in range(1, 4):
        bm.fork(0, j)
    assert bm.ref[:3] == [4, 4, 4]
    pairs = []
    for j in range(4):
        slot, cow = bm.append_slot(j)
        if cow:
            pairs.append(cow)
        assert slot % 4 == 2
    assert pairs == [(2, 3), (2, 4), (2, 5)]
    assert bm.block_table(3) == [0, 1, 2]   # last sharer kept the original
    assert bm.ref[:6] == [4, 4, 1, 1, 1, 1]
    _invariants(bm)
    for j in range(4):
        bm.free_seq(j)
    assert sorted(bm.free) == list(range(64))


def test_cow_count_for_sampling_recipe():
    """Per prompt, samples 0..6 copy the shared partial block, sample 7 writes in place."""
    w = W.parallel_sampling(seed=1, num_prompts=3, num_samples=8, max_tail=40)
    bm = BlockManagerModel(w.num_blocks, w.shape.block_size, w.free_order)
    pairs_first = None
    for op in W.sampling_ops(w):
        if op[0] == "add":
            bm.add_seq(op[1], op[2])
        elif op[0] == "fork":
            bm.fork(op[1], op[2])
        elif op[0] == "append":
            pairs = [c for c in (bm.append_slot(s)[1] for s in op[1]) if c]
            if pairs_first is None:
                pairs_first = pairs
            else:
                assert pairs == []
    assert len(pairs_first) == 3 * 7
    _invariants(bm)


def test_exhaustion_leaves_state_unchanged():
    bm = BlockManagerModel(3, 4, [2, 0, 1])
    bm.add_seq(0, 8)
    snap = copy.deepcopy((list(bm.free), bm.ref, bm.tables, bm.lens))
    with pytest.raises(NoFreeBlocks):
        bm.add_seq(1, 9)
    assert snap == (list(bm.free), bm.ref, bm.tables, bm.lens)
    bm.add_seq(1, 4)
    snap = copy.deepcopy((list(bm.free), bm.ref, bm.tables, bm.lens))
    with pytest.raises(NoFreeBlocks):
        bm.append_slot(1)                  # block full, pool empty
    assert snap == (list(bm.free), bm.ref, bm.tables, bm.lens)
    with pytest.raises(UnknownSeq):
        bm.free_seq(7)
    with pytest.raises(OracleError):
        bm.add_seq(0, 1)


def test_cow_exhaustion_leaves_state_unchanged():
    bm = BlockManagerModel(1, 4, [0])
    bm.add_seq(0, 2)
    bm.fork(0, 1)
    snap = copy.deepcopy((list(bm.free), bm.ref, bm.tables, bm.lens))
    with pytest.raises(NoFreeBlocks):
        bm.append_slot(0)
    assert snap == (list(bm.free), bm.ref, bm.tables, bm.lens)


def test_fragmentation_free_blocks_serve_anyone():
    """P1 "为什么 Paged Attention 如此高效": scattered free blocks still serve a new
    request whose size equals their sum (no external waste)."""
    bm = BlockManagerModel(8, 2, list(range(8)))
    for s in range(8):
        bm.add_seq(s, 2)
    for s in (1, 3, 4, 6):
        bm.free_seq(s)
    bm.add_seq(100, 8)
    assert sorted(bm.block_table(100)) == [1, 3, 4, 6]
    assert bm.stats()["internal_waste"] == 0
