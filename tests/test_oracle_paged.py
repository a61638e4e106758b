"""Pins for the oracle scatter / gather / block copy and the replay (no GPU).

P1 = page "Paged Attention：大模型推理显存优化的核心方案" ("什么是 Paged
Attention？": blocks need not be contiguous); P2 = page "PagedAttention：操作系统级
KV 缓存虚拟内存管理" (§2.3, §3.2, §3.4, §五).
"""
import numpy as np
import pytest
import torch

from oracle import paged
from oracle.replay import OracleRun
from paged_kv_cache_361_b200 import workloads as W


def _same_bits(a, b):
    return a.shape == b.shape and torch.equal(a.view(torch.int16 if a.dtype == torch.bfloat16 else torch.int32),
                                              b.view(torch.int16 if b.dtype == torch.bfloat16 else torch.int32))


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gather_equals_contiguous_history(bs, dtype):
    """Physical placement is invisible: the table walk returns the history bitwise,
    for any block size and any permutation of physical ids."""
    sh = W.Shape(4, 2, 8, bs, dtype)
    w = W.random_small(seed=bs, num_seqs=5, shape=sh, max_len=3 * bs + 5)
    run = OracleRun(sh, w.num_blocks, w.free_order).run(W.simple_ops(w))
    for s in range(w.num_seqs):
        for which in "kv":
            assert _same_bits(run.paged_rows(s, which), run.history(s, which))
            assert _same_bits(run.history(s, which), w.history(s, which))


def test_gather_invariant_to_physical_permutation():
    sh = W.Shape(2, 2, 4, 4, "f32")
    w = W.random_small(seed=7, num_seqs=4, shape=sh, max_len=20)
    outs = []
    for perm_seed in range(3):
        order = np.random.default_rng(perm_seed).permutation(w.num_blocks)
        run = OracleRun(sh, w.num_blocks, order).run(W.simple_ops(w))
        q = w.query()
        outs.append([run.attend(s, q[s], w.scale, use_pool=True) for s in range(w.num_seqs)])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a, b)


def test_padding_is_never_read():
    """P2 §3.2.1: unfilled slots of the last block are padding; a NaN there must not
    reach any gathered row."""
    w = W.tiny_fp32()
    run = OracleRun(w.shape, w.num_blocks, w.free_order, pool_fill=float("nan")).run(W.simple_ops(w))
    assert torch.isnan(run.pool["k"]).any()
    for s in range(w.num_seqs):
        assert not torch.isnan(run.paged_rows(s, "k")).any()
        out = run.attend(s, w.query()[s], w.scale, use_pool=True)
        assert np.isfinite(out).all()


def test_copy_blocks_is_a_bit_copy():
    pool = paged.new_pool(6, 2, 4, 8, torch.bfloat16, 0.0)
    pool.copy_(torch.randn(pool.shape).to(torch.bfloat16))
    before = pool.clone()
    paged.copy_blocks(pool, [(1, 4), (2, 5)])
    assert torch.equal(pool[4], before[1]) and torch.equal(pool[5], before[2])
    for b in (0, 1, 2, 3):
        assert torch.equal(pool[b], before[b])


def test_scatter_skips_minus_one():
    pool = paged.new_pool(2, 1, 2, 2, torch.float32, 0.0)
    paged.scatter(pool, torch.ones(3, 1, 2), [1, -1, 2])
    assert pool.sum().item() == 4.0
    assert pool[0, 0, 1].tolist() == [1.0, 1.0] and pool[1, 0, 0].tolist() == [1.0, 1.0]


def test_sampling_siblings_share_prefix_and_stay_independent():
    """P2 §3.4 / §五: forks read the same prefix rows; copy-on-write keeps one
    sample's writes out of its siblings' rows."""
    w = W.parallel_sampling(seed=2, num_prompts=2, num_samples=4, prefix_len=21, max_tail=9)
    run = OracleRun(w.shape, w.num_blocks, w.free_order)
    ops = W.sampling_ops(w)
    for op in ops:
        run.apply(op)
    pre = w.extra["prefix_len"]
    for s in range(8):
        for which in "kv":
            hist = W.sampling_history(w, s, which)
            got = run.paged_rows(s, which)
            assert _same_bits(got, hist)
            assert _same_bits(got[:pre], W.prefix_values(w, s // 4, which))
    n_pairs = sum(len(r["pairs"]) for r in run.records if r["kind"] == "append")
    assert n_pairs == 2 * 3


def test_identical_siblings_identical_outputs():
    """Two samples with identical tails and queries produce identical outputs."""
    sh = W.Shape(2, 1, 8, 4, "f32")
    bm_run = OracleRun(sh, 32, list(range(32)))
    pre_k = torch.randn(6, 1, 8)
    pre_v = torch.randn(6, 1, 8)
    bm_run.apply(("add", 0, 6, lambda which, device="cpu": pre_k if which == "k" else pre_v))
    bm_run.apply(("fork", 0, 1))
    tail = {"k": torch.randn(1, 1, 8), "v": torch.randn(1, 1, 8)}
    bm_run.apply(("append", [0, 1], lambda which, device="cpu": torch.cat([tail[which], tail[which]])))
    q = torch.randn(2, 8)
    a = bm_run.attend(0, q, 0.3, use_pool=True)
    b = bm_run.attend(1, q, 0.3, use_pool=True)
    assert np.array_equal(a, b)
    assert bm_run.bm.block_table(0)[1] != bm_run.bm.block_table(1)[1]


def test_replay_batching_matches_history():
    tr = W.continuous_batching(seed=5, num_live=6, steps=30, num_blocks=600, p_finish=0.1)
    run = OracleRun(tr.shape, tr.num_blocks, tr.free_order)
    ops = W.batching_ops(tr)
    for op in ops:
        run.apply(op)
    for s in run.bm.tables:
        for which in "kv":
            assert _same_bits(run.paged_rows(s, which), run.history(s, which))
