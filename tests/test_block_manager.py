"""The C++ block manager (through the C ABI) against the oracle model, bit-exact:
slots, copy-on-write pairs, tables, reference counts, free lists and waste
statistics after the operation scripts of every workload. No GPU needed."""
import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel
from paged_kv_cache_361_b200 import binding as B
from paged_kv_cache_361_b200 import workloads as W


def _replay_both(num_blocks, block_size, free_order, ops, check_every=1, check_free_every=50):
    cpp = B.BlockManager(num_blocks, block_size, free_order)
    ref = BlockManagerModel(num_blocks, block_size, free_order)
    live = set()
    n_pairs = 0
    for i, op in enumerate(ops):
        kind = op[0]
        if kind == "add":
            a = cpp.add_seq(op[1], op[2])
            b = ref.add_seq(op[1], op[2])
            assert a.tolist() == b
            live.add(op[1])
        elif kind == "fork":
            cpp.fork(op[1], op[2])
            ref.fork(op[1], op[2])
            live.add(op[2])
        elif kind == "append":
            slots, pairs = cpp.append_slots(op[1])
            rs, rp = [], []
            for s in op[1]:
                sl, cow = ref.append_slot(s)
                rs.append(sl)
                if cow:
                    rp.append(list(cow))
            assert slots.tolist() == rs
            assert pairs.tolist() == rp
            n_pairs += len(rp)
        elif kind == "free":
            cpp.free_seq(op[1])
            ref.free_seq(op[1])
            live.discard(op[1])
        if i % check_every == 0 or i == len(ops) - 1:
            for s in live:
                t, L = cpp.block_table(s)
                assert t.tolist() == ref.block_table(s) and L == ref.lens[s]
        if i % check_free_every == 0 or i == len(ops) - 1:
            assert cpp.free_list().tolist() == list(ref.free)
            st = ref.stats()
            got = cpp.stats()
            for k in ("free_blocks", "used_slots", "allocated_slots", "internal_waste"):
                assert got[k] == st[k], k
    for b in range(num_blocks):
        assert cpp.refcount(b) == ref.ref[b]
    return cpp, ref, n_pairs


def test_tiny_fp32_script():
    w = W.tiny_fp32()
    cpp, ref, _ = _replay_both(w.num_blocks, w.shape.block_size, w.free_order, W.simple_ops(w))
    # sequence 0 is the page's 10-token example plus the appended token
    assert len(ref.block_table(0)) == 3 and ref.lens[0] == 11


def test_llama2_7b_mha_script():
    w = W.llama2_7b_mha()
    _replay_both(w.num_blocks, w.shape.block_size, w.free_order, W.simple_ops(w), check_free_every=1)


def test_long_context_script():
    w = W.long_context_split()
    _replay_both(w.num_blocks, w.shape.block_size, w.free_order, W.simple_ops(w))


def test_parallel_sampling_script():
    w = W.parallel_sampling()
    _, _, n_pairs = _replay_both(w.num_blocks, w.shape.block_size, w.free_order, W.sampling_ops(w),
                                 check_every=64, check_free_every=200)
    assert n_pairs == 8 * 7


def test_continuous_batching_script():
    tr = W.continuous_batching()
    _replay_both(tr.num_blocks, tr.shape.block_size, tr.free_order, W.batching_ops(tr), check_every=25,
                 check_free_every=300)


def test_batched_append_equals_sequential_with_duplicates_and_cow():
    rng = np.random.default_rng(0)
    for trial in range(30):
        bs = int(rng.choice([1, 2, 4, 8]))
        nb = 200
        order = rng.permutation(nb)
        a = B.BlockManager(nb, bs, order)
        b = BlockManagerModel(nb, bs, order)
        a.add_seq(0, int(rng.integers(0, 3 * bs)))
        b.add_seq(0, a.block_table(0)[1])
        for c in range(1, 4):
            a.fork(0, c)
            b.fork(0, c)
        ids = rng.integers(0, 4, size=12).tolist()
        slots, pairs = a.append_slots(ids)
        rs, rp = [], []
        for s in ids:
            sl, cow = b.append_slot(s)
            rs.append(sl)
            if cow:
                rp.append(list(cow))
        assert slots.tolist() == rs and pairs.tolist() == rp
        assert a.free_list().tolist() == list(b.free)


def test_errors_leave_state_unchanged():
    bm = B.BlockManager(4, 4, [3, 2, 1, 0])
    bm.add_seq(1, 8)
    bm.fork(1, 2)
    before = (bm.free_list().tolist(), bm.block_table(1)[0].tolist(), bm.block_table(2)[0].tolist())
    with pytest.raises(B.PagedAttnError) as e:
        bm.add_seq(3, 9)
    assert e.value.status == B.PA_ERR_NO_FREE_BLOCKS
    with pytest.raises(B.PagedAttnError) as e:
        bm.add_seq(1, 1)
    assert e.value.status == B.PA_ERR_SEQ_EXISTS
    with pytest.raises(B.PagedAttnError) as e:
        bm.free_seq(9)
    assert e.value.status == B.PA_ERR_UNKNOWN_SEQ
    with pytest.raises(B.PagedAttnError) as e:
        bm.fork(9, 10)
    assert e.value.status == B.PA_ERR_UNKNOWN_SEQ
    # a batch needing 3 fresh blocks with 2 free fails whole
    with pytest.raises(B.PagedAttnError) as e:
        bm.append_slots([1, 2, 1, 2, 1, 2, 1, 2, 1])
    assert e.value.status == B.PA_ERR_NO_FREE_BLOCKS
    assert before == (bm.free_list().tolist(), bm.block_table(1)[0].tolist(), bm.block_table(2)[0].tolist())
    with pytest.raises(B.PagedAttnError):
        B.BlockManager(4, 4, [0, 1, 1, 2])      # not a permutation
    with pytest.raises(B.PagedAttnError) as e:
        bm.block_tables([1, 2], cap=1)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_block_tables_padding():
    bm = B.BlockManager(10, 4)
    bm.add_seq(5, 9)
    bm.add_seq(6, 1)
    t, lens = bm.block_tables([6, 5], cap=4, pad=-1)
    assert t.tolist() == [[3, -1, -1, -1], [0, 1, 2, -1]] and lens.tolist() == [1, 9]


def _replay_prefix(tr_or_ops, num_blocks, bs, order, ops):
    from oracle.prefix_cache import PrefixCachingModel
    cpp = B.BlockManager(num_blocks, bs, order)
    ref = PrefixCachingModel(num_blocks, bs, order)
    live = set()
    for op in ops:
        if op[0] == "add_cached":
            a, na = cpp.add_seq_cached(op[1], op[2])
            b, nb = ref.add_seq_cached(op[1], op[2])
            assert a.tolist() == b and na == nb
            live.add(op[1])
        elif op[0] == "append":
            slots, pairs = cpp.append_slots(op[1])
            rs = [ref.append_slot(s)[0] for s in op[1]]
            assert slots.tolist() == rs
        elif op[0] == "free":
            cpp.free_seq(op[1])
            ref.free_seq(op[1])
            live.discard(op[1])
        for s in live:
            assert cpp.block_table(s)[0].tolist() == ref.block_table(s)
        assert cpp.free_list().tolist() == list(ref.free)
        st = cpp.prefix_stats()
        assert st == ref.prefix_stats()
    for b in range(num_blocks):
        assert cpp.refcount(b) == ref.ref[b]
    return cpp, ref


def test_prefix_cache_trace_bit_exact():
    tr = W.prefix_caching()
    cpp, ref = _replay_prefix(tr, tr.num_blocks, tr.shape.block_size, tr.free_order, W.prefix_ops(tr))
    st = ref.prefix_stats()
    assert st["hit_tokens"] > 0 and st["cached_blocks"] > 0


def test_prefix_cache_random_stress_with_eviction():
    rng = np.random.default_rng(7)
    for trial in range(20):
        bs = int(rng.choice([1, 2, 4]))
        nb = int(rng.integers(8, 40))
        order = rng.permutation(nb)
        prefixes = [rng.integers(0, 5, size=int(rng.integers(0, 3 * bs + 2))).tolist() for _ in range(3)]
        ops, live, nid = [], [], 0
        for step in range(60):
            u = rng.random()
            if u < 0.4 or not live:
                toks = prefixes[int(rng.integers(0, 3))] + rng.integers(0, 5, size=int(rng.integers(0, 2 * bs))).tolist()
                ops.append(("add_cached", nid, toks))
                live.append(nid)
                nid += 1
            elif u < 0.7:
                ops.append(("append", [live[int(rng.integers(0, len(live)))]]))
            else:
                ops.append(("free", live.pop(int(rng.integers(0, len(live))))))
        # run until the first failure on the oracle side, which must fail identically in C++
        from oracle.prefix_cache import PrefixCachingModel
        from oracle.block_manager import NoFreeBlocks
        cpp = B.BlockManager(nb, bs, order)
        ref = PrefixCachingModel(nb, bs, order)
        for op in ops:
            try:
                if op[0] == "add_cached":
                    exp = ref.add_seq_cached(op[1], op[2])
                elif op[0] == "append":
                    exp = ref.append_slot(op[1][0])[0]
                else:
                    exp = ref.free_seq(op[1])
                ok = True
            except NoFreeBlocks:
                ok = False
            if op[0] == "add_cached":
                if ok:
                    got = cpp.add_seq_cached(op[1], op[2])
                    assert got[0].tolist() == exp[0] and got[1] == exp[1]
                else:
                    with pytest.raises(B.PagedAttnError):
                        cpp.add_seq_cached(op[1], op[2])
                    break
            elif op[0] == "append":
                if ok:
                    assert cpp.append_slot(op[1][0])[0] == exp
                else:
                    with pytest.raises(B.PagedAttnError):
                        cpp.append_slot(op[1][0])
                    break
            else:
                cpp.free_seq(op[1])
            assert cpp.free_list().tolist() == list(ref.free)
            assert cpp.prefix_stats() == ref.prefix_stats()


def test_batched_append_stress_one_manager():
    """Many batched appends on one manager (its batch scratch reused across
    calls): random batches with repeated ids over forked sequences, frees and
    adds in between, and batches that must fail whole (too few free blocks, an
    unknown id); after every call slots, pairs, tables and the free list equal
    the oracle's sequential appends, and a failed batch changes nothing."""
    import copy
    from oracle.block_manager import NoFreeBlocks, UnknownSeq
    rng = np.random.default_rng(11)
    nb, bs = 48, 4
    order = rng.permutation(nb)
    a = B.BlockManager(nb, bs, order)
    m = BlockManagerModel(nb, bs, order)
    next_id = 0
    live = []
    for rnd in range(400):
        op = rng.random()
        if (op < 0.15 or not live) and len(live) < 10:
            n = int(rng.integers(0, 3 * bs))
            try:
                m2 = copy.deepcopy(m)
                m2.add_seq(next_id, n)
            except NoFreeBlocks:
                with pytest.raises(B.PagedAttnError):
                    a.add_seq(next_id, n)
                continue
            a.add_seq(next_id, n)
            m = m2
            live.append(next_id)
            next_id += 1
        elif op < 0.25 and len(live) < 10:
            parent = int(rng.choice(live))
            a.fork(parent, next_id)
            m.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.35 and len(live) > 1:
            s = int(live.pop(int(rng.integers(len(live)))))
            a.free_seq(s)
            m.free_seq(s)
        else:
            ids = [int(x) for x in rng.choice(live, size=int(rng.integers(1, 9)))]
            if rng.random() < 0.05:
                ids.insert(int(rng.integers(len(ids) + 1)), 10 ** 6)   # unknown id: the batch fails whole
            m2 = copy.deepcopy(m)
            rs, rp, err = [], [], None
            try:
                for s in ids:
                    sl, cow = m2.append_slot(s)
                    rs.append(sl)
                    if cow:
                        rp.append(list(cow))
            except (NoFreeBlocks, UnknownSeq) as e:
                err = e
            before = (a.free_list().tolist(), [a.block_table(s)[0].tolist() for s in live])
            if err is not None:
                with pytest.raises(B.PagedAttnError) as e:
                    a.append_slots(ids)
                # every id is looked up before the blocks are counted: an unknown id wins
                assert e.value.status == (B.PA_ERR_UNKNOWN_SEQ if 10 ** 6 in ids else B.PA_ERR_NO_FREE_BLOCKS)
                assert before == (a.free_list().tolist(), [a.block_table(s)[0].tolist() for s in live])
                continue
            slots, pairs = a.append_slots(ids)
            m = m2
            assert slots.tolist() == rs and pairs.tolist() == rp, rnd
        assert a.free_list().tolist() == list(m.free), rnd
        for s in live:
            assert a.block_table(s)[0].tolist() == m.block_table(s), (rnd, s)
