"""GPU parity on the five workloads at full size.

  tiny_fp32            in test_gpu_decode (whole pool and every output)
  llama2_7b_mha        64 seqs x 32 heads, lengths 129..2049: every output row,
                       every sequence's cached rows bitwise
  parallel_sampling    8 prompts x 8 samples, CoW at the first tail step:
                       56 pairs, every output row, every cached row
  continuous_batching  200 steps over a 200k-block pool: slots and tables at
                       every step; all outputs at 5 steps, 2 sequences at
                       every other step
  long_context_split   4 seqs up to 131073 tokens, 512-token partitions (and
                       no split, and the library's choice): every output row
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_361_b200 import binding as B
from paged_kv_cache_361_b200 import workloads as W
from tests.parity import Replay

pytestmark = pytest.mark.gpu


def test_llama2_7b_mha():
    w = W.llama2_7b_mha()
    r = Replay(w.shape, w.num_blocks, w.free_order, w.scale, keep_pool=False).run(W.simple_ops(w))
    r.check_pool_rows()
    r.check_outputs()


def test_parallel_sampling():
    w = W.parallel_sampling()
    r = Replay(w.shape, w.num_blocks, w.free_order, w.scale, keep_pool=False)
    r.run(W.sampling_ops(w, batch_tail_steps=True))
    assert r.n_pairs == 56
    r.check_pool_rows()
    r.check_outputs()
    # siblings share the prefix rows bitwise (CoW left the shared blocks alone)
    pre = w.extra["prefix_len"]
    for p in range(8):
        for j in range(8):
            hist = W.sampling_history(w, p * 8 + j, "k")
            assert torch.equal(hist[:pre].view(torch.int16), W.prefix_values(w, p, "k").view(torch.int16))


def test_continuous_batching():
    tr = W.continuous_batching()
    r = Replay(tr.shape, tr.num_blocks, tr.free_order, 1.0 / np.sqrt(128), keep_pool=False)
    rng = np.random.default_rng(0)
    step = 0
    full_steps = {0, 1, 2, 100, 199}
    for op in W.batching_ops(tr):
        r.apply(op)
        if op[0] == "decode":
            if step in full_steps:
                r.check_outputs()
            else:
                r.check_outputs(seqs=set(rng.choice(len(op[1]), 2, replace=False).tolist()))
            r.decodes.clear()
            step += 1
    assert step == 200
    st, info = B.pa_get_device_error()
    assert st == B.PA_OK, (st, info)
    r.check_pool_rows(seqs=list(r.cache.lens)[:16])


@pytest.mark.parametrize("P", [512, 0, -1])
def test_long_context_split(P):
    w = W.long_context_split()
    r = Replay(w.shape, w.num_blocks, w.free_order, w.scale, partition_tokens=P, keep_pool=False)
    r.run(W.simple_ops(w))
    r.check_outputs()
    if P == 512:
        r.check_pool_rows()


def test_prefix_caching_trace():
    """Requests sharing system prompts: cached whole blocks are reused (their rows
    are not written again) and evicted under a small pool; slots, tables and every
    decode output match the oracle."""
    tr = W.prefix_caching()
    r = Replay(tr.shape, tr.num_blocks, tr.free_order, 1.0 / np.sqrt(128), keep_pool=True)
    for op in W.prefix_ops(tr):
        r.apply(op)
        if op[0] == "decode":
            r.check_outputs()
            r.decodes.clear()
    assert r.n_cached > 0
    st, info = B.pa_get_device_error()
    assert st == B.PA_OK, (st, info)
    r.check_pool_rows()
    assert r.cache.bm.prefix_stats() == r.oracle.bm.prefix_stats()
