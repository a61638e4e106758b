"""Swapping sequences between the device pool and host blocks (P2 = page
"PagedAttention：操作系统级 KV 缓存虚拟内存管理", §五 page replacement, §八 GPU/CPU
tiers): the oracle's conventions, and the C++ manager bit-exact against them."""
import numpy as np
import pytest

from oracle.block_manager import NoFreeBlocks
from oracle.swap import SwappingModel
from paged_kv_cache_361_b200 import binding as B


def test_oracle_swap_out_releases_and_swap_in_restores():
    m = SwappingModel(6, 2, list(range(6)), host_blocks=4)
    m.add_seq(1, 5)                       # blocks 0, 1, 2
    m.add_seq(2, 2)                       # block 3
    pairs = m.swap_out(1)
    assert pairs == [(0, 0), (1, 1), (2, 2)]
    assert list(m.free) == [4, 5, 0, 1, 2] and list(m.host_free) == [3]
    m.add_seq(3, 4)                       # reuses 4, 5
    back = m.swap_in(1)                   # fresh blocks 0, 1, 2 from the free list
    assert back == [(0, 0), (1, 1), (2, 2)] and m.lens[1] == 5
    assert list(m.host_free) == [3, 0, 1, 2]
    m.free_seq(3)                         # free: 4, 5
    m.add_seq(4, 1)                       # block 4
    m.swap_out(4)                         # block 4 released
    m.add_seq(5, 4)                       # blocks 5, 4: the pool is full
    with pytest.raises(NoFreeBlocks):
        m.swap_in(4)


def test_oracle_shared_blocks_stay_for_other_holder():
    m = SwappingModel(8, 2, list(range(8)), host_blocks=8)
    m.add_seq(1, 4)
    m.fork(1, 2)
    m.swap_out(1)
    assert m.ref[0] == 1 and m.ref[1] == 1       # still held by sequence 2
    assert m.block_table(2) == [0, 1]
    m.free_seq(1)                                 # frees the host copy
    assert len(m.host_free) == 8


def test_oracle_swap_errors_leave_state():
    m = SwappingModel(4, 2, list(range(4)), host_blocks=1)
    m.add_seq(1, 4)
    snap = (list(m.free), list(m.host_free), dict(m.tables))
    with pytest.raises(NoFreeBlocks):
        m.swap_out(1)
    assert snap == (list(m.free), list(m.host_free), dict(m.tables))


def _both(nb, hb, bs, order):
    a = B.BlockManager(nb, bs, order)
    a.set_host_blocks(hb)
    return a, SwappingModel(nb, bs, order, host_blocks=hb)


def _call_both(cpp_fn, ref_fn):
    """Run the same call on both; both succeed with the same result or both
    refuse for lack of blocks."""
    try:
        exp = ref_fn()
    except NoFreeBlocks:
        with pytest.raises(B.PagedAttnError) as e:
            cpp_fn()
        assert e.value.status == B.PA_ERR_NO_FREE_BLOCKS
        return None, False
    return (cpp_fn(), exp), True


def test_swap_cpp_matches_oracle_random():
    rng = np.random.default_rng(3)
    for trial in range(25):
        bs = int(rng.choice([1, 2, 4]))
        nb, hb = int(rng.integers(6, 30)), int(rng.integers(2, 20))
        order = rng.permutation(nb)
        cpp, ref = _both(nb, hb, bs, order)
        live, out, nid = [], [], 0
        for step in range(80):
            u = rng.random()
            if u < 0.25 or not (live or out):
                n = int(rng.integers(0, 3 * bs))
                r, ok = _call_both(lambda: cpp.add_seq(nid, n), lambda: ref.add_seq(nid, n))
                if ok:
                    assert r[0].tolist() == r[1]
                    live.append(nid)
                    nid += 1
            elif u < 0.45 and live:
                s_ = live[int(rng.integers(0, len(live)))]
                r, ok = _call_both(lambda: cpp.append_slot(s_)[0], lambda: ref.append_slot(s_)[0])
                if ok:
                    assert r[0] == r[1]
            elif u < 0.6 and live:
                s_ = live[int(rng.integers(0, len(live)))]
                r, ok = _call_both(lambda: cpp.swap_out(s_), lambda: ref.swap_out(s_))
                if ok:
                    assert [tuple(x) for x in r[0].tolist()] == r[1]
                    live.remove(s_)
                    out.append(s_)
            elif u < 0.8 and out:
                s_ = out[int(rng.integers(0, len(out)))]
                r, ok = _call_both(lambda: cpp.swap_in(s_), lambda: ref.swap_in(s_))
                if ok:
                    assert [tuple(x) for x in r[0].tolist()] == r[1]
                    out.remove(s_)
                    live.append(s_)
            elif live or out:
                pool = live + out
                s_ = pool[int(rng.integers(0, len(pool)))]
                ref.free_seq(s_)
                cpp.free_seq(s_)
                (live if s_ in live else out).remove(s_)
            assert cpp.free_list().tolist() == list(ref.free)
            for s_ in live:
                assert cpp.block_table(s_)[0].tolist() == ref.block_table(s_)
        for b in range(nb):
            assert cpp.refcount(b) == ref.ref[b]


def test_swapped_sequence_is_not_live():
    cpp = B.BlockManager(4, 2)
    cpp.set_host_blocks(4)
    cpp.add_seq(1, 3)
    cpp.swap_out(1)
    with pytest.raises(B.PagedAttnError) as e:
        cpp.append_slot(1)
    assert e.value.status == B.PA_ERR_UNKNOWN_SEQ
    with pytest.raises(B.PagedAttnError) as e:
        cpp.add_seq(1, 1)
    assert e.value.status == B.PA_ERR_SEQ_EXISTS
    with pytest.raises(B.PagedAttnError):
        cpp.set_host_blocks(8)          # not while a sequence is swapped out
    cpp.free_seq(1)
    cpp.set_host_blocks(8)
