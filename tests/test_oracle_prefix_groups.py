"""Pins of the shared-prefix grouping oracle (P2 §3.4: shared prefixes are the
same physical blocks) on hand-worked block tables, then the C++ block
manager's pa_bm_prefix_groups against the oracle on random fork families."""
import numpy as np
import pytest

from oracle.prefix_groups import prefix_groups
from paged_kv_cache_361_b200 import binding as B


def test_two_forks_of_one_prompt():
    # 100 tokens in blocks of 16: 6 whole blocks (96 tokens) shared, cut to 64
    t = [[7, 3, 9, 1, 4, 2, 8], [7, 3, 9, 1, 4, 2, 5]]
    assert prefix_groups(t, [101, 101], 16, 16, 64) == ([0, 2], [0, 1], [64], [64, 64])
    # alignment 16 keeps all 6 whole blocks
    assert prefix_groups(t, [101, 101], 16, 16, 16) == ([0, 2], [0, 1], [96], [96, 96])


def test_copy_on_write_inside_the_prefix_stops_it():
    # the third entry differs: only 2 blocks (32 tokens) in common
    t = [[7, 3, 9, 1, 4], [7, 3, 6, 1, 4]]
    assert prefix_groups(t, [80, 80], 16, 16, 16) == ([0, 2], [0, 1], [32], [32, 32])
    assert prefix_groups(t, [80, 80], 16, 16, 64) == ([0], [], [], [0, 0])   # cut to 0: dropped


def test_shortest_member_bounds_the_prefix():
    t = [[1, 2, 3, 4, 5], [1, 2, 3, 4, 5]]
    # member 1 holds 50 tokens: 3 whole blocks, the partly filled 4th is never shared
    assert prefix_groups(t, [80, 50], 16, 16, 16) == ([0, 2], [0, 1], [48], [48, 48])


def test_lone_and_short_sequences_take_no_part():
    t = [[5, 6], [9, 1], [5, 6], [2]]
    lens = [32, 32, 32, 10]          # sequence 3 has no whole block
    assert prefix_groups(t, lens, 16, 16, 16) == ([0, 2], [0, 2], [32], [32, 0, 32, 0])


def test_group_size_cut_in_batch_order():
    t = [[4, 8]] * 5
    off, mem, pre, sp = prefix_groups(t, [32] * 5, 16, 2, 16)
    assert off == [0, 2, 4] and mem == [0, 1, 2, 3] and pre == [32, 32] and sp == [32, 32, 32, 32, 0]


def test_keys_in_order_of_first_appearance():
    t = [[3, 1], [8, 1], [3, 1], [8, 1]]
    off, mem, pre, _ = prefix_groups(t, [32] * 4, 16, 8, 16)
    assert mem == [0, 2, 1, 3] and off == [0, 2, 4]


@pytest.mark.parametrize("seed", range(6))
def test_cpp_prefix_groups_match_oracle(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([8, 16, 32]))
    bm = B.BlockManager(6000, bs, rng.permutation(6000))
    ids = []
    for fam in range(int(rng.integers(2, 7))):
        root = 1000 * fam
        bm.add_seq(root, int(rng.integers(1, 900)))
        kids = [root]
        for j in range(int(rng.integers(0, 12))):
            bm.fork(root, root + j + 1)
            kids.append(root + j + 1)
        ids += kids
    ids = [int(x) for x in rng.permutation(ids)]
    for _ in range(int(rng.integers(0, 40))):      # private suffixes, with copy-on-write
        sub = [s for s in ids if rng.random() < 0.7]
        bm.append_slots(sub)
    tables = [bm.block_table(s)[0].tolist() for s in ids]
    lens = [bm.block_table(s)[1] for s in ids]
    for max_group in (2, 8, 64):
        for align in (bs, 64):
            off, mem, pre, sp, mp = bm.prefix_groups(ids, max_group, align)
            ro, rm, rp, rsp = prefix_groups(tables, lens, bs, max_group, align)
            assert off.tolist() == ro and mem.tolist() == rm and pre.tolist() == rp and sp.tolist() == rsp
            assert mp == max(rp, default=0)


def test_cpp_prefix_groups_errors():
    bm = B.BlockManager(16, 4)
    bm.add_seq(1, 8)
    with pytest.raises(B.PagedAttnError) as e:
        bm.prefix_groups([1, 2], 4)
    assert e.value.status == B.PA_ERR_UNKNOWN_SEQ
    with pytest.raises(B.PagedAttnError) as e:
        bm.prefix_groups([1], 0)
    assert e.value.status == B.PA_ERR_INVALID_ARG
    off, mem, pre, sp, mp = bm.prefix_groups([], 4)
    assert off.tolist() == [0] and len(mem) == 0 and mp == 0


def test_cpp_longest_first():
    """pa_bm_longest_first: rows by decreasing (tokens - skip), ties in batch
    order; unknown ids and missing arrays are errors."""
    bm = B.BlockManager(64, 4)
    for sid, n in ((10, 5), (11, 9), (12, 9), (13, 1), (14, 12)):
        bm.add_seq(sid, n)
    assert bm.longest_first([10, 11, 12, 13, 14]).tolist() == [4, 1, 2, 0, 3]
    # spans 5-0, 9-8, 9-0, 1-0, 12-12 -> 9, 5, 1, 1, 0
    assert bm.longest_first([10, 11, 12, 13, 14], [0, 8, 0, 0, 12]).tolist() == [2, 0, 1, 3, 4]
    assert bm.longest_first([]).tolist() == []
    with pytest.raises(B.PagedAttnError) as e:
        bm.longest_first([10, 99])
    assert e.value.status == B.PA_ERR_UNKNOWN_SEQ
    with pytest.raises(ValueError):
        bm.longest_first([10, 11], [0])
