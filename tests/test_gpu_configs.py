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


def test_parallel_sampling_cascade():
    """Shared-prefix decode on the parallel-sampling workload: each prompt's
    prefix blocks are read once for its 8 samples; outputs match the oracle."""
    w = W.parallel_sampling()
    r = Replay(w.shape, w.num_blocks, w.free_order, w.scale, keep_pool=False)
    ops = W.sampling_ops(w, batch_tail_steps=True)
    for op in ops[:-1]:
        r.apply(op)
    ids, qsrc = ops[-1][1], ops[-1][2]
    q = qsrc()
    r.oracle.apply(ops[-1])
    out = r.cache.decode_cascade(ids, q.cuda(), w.scale).cpu()
    st, info = B.pa_get_device_error()
    assert st == B.PA_OK, (st, info)
    offs, members, prefix, seq_prefix, _ = r.cache.shared_prefix_groups(ids, 16)
    assert len(prefix) == 8 and (prefix == 960).all()      # 62 shared blocks of 16 -> 960 tokens
    r.decodes.append((list(ids), q, out))
    r.check_outputs()


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_cascade_random_groups(G):
    """Forked families with random suffixes (and lone sequences) against pa_decode."""
    from paged_kv_cache_361_b200 import PagedKVCache
    rng = np.random.default_rng(G)
    hkv, D, bs = 2, 128, 16
    cache = PagedKVCache(4000, hkv, bs, D, torch.bfloat16, "cuda", rng.permutation(4000), fill=float("nan"))
    g = torch.Generator().manual_seed(G)
    ids = []
    for fam in range(5):
        root = fam * 100
        n0 = int(rng.integers(64, 700))
        cache.add_sequence(root, torch.randn(n0, hkv, D, generator=g).bfloat16().cuda(),
                           torch.randn(n0, hkv, D, generator=g).bfloat16().cuda())
        ids.append(root)
        for j in range(1, int(rng.integers(1, 64 // G + 3))):
            cache.fork(root, root + j)
            ids.append(root + j)
    for _ in range(int(rng.integers(1, 40))):       # private suffixes
        k = torch.randn(len(ids), hkv, D, generator=g).bfloat16().cuda()
        cache.append(ids, k, k)
    q = torch.randn(len(ids), hkv * G, D, generator=g).bfloat16().cuda()
    a = cache.decode(ids, q, D ** -0.5)
    b = cache.decode_cascade(ids, q, D ** -0.5)
    assert B.pa_get_device_error()[0] == B.PA_OK
    assert float((a - b).abs().max()) <= 2e-3


@pytest.mark.parametrize("fmt,G,D,bs", [("e4m3", 1, 128, 16), ("e4m3", 8, 128, 16), ("int8", 4, 128, 16),
                                          ("int8", 2, 64, 16), ("e4m3", 4, 64, 16), ("int8", 8, 128, 16),
                                          ("e4m3", 2, 128, 8), ("int8", 1, 64, 8), ("int8", 4, 128, 32),
                                          ("e4m3", 8, 64, 32)])
def test_cascade_8bit_cache(fmt, G, D, bs):
    """Shared-prefix decode over an 8-bit cache: forked families with private
    suffixes and lone sequences; equal to pa_decode on the same cache, and to
    the oracle's attention over the dequantised rows on sampled sequences."""
    from oracle import fp8, int8
    from oracle.attention import decode_attention
    from paged_kv_cache_361_b200 import PagedKVCache
    codec, dt, ks, vs = ((fp8, torch.float8_e4m3fn, 4.0 / 448, 3.0 / 448) if fmt == "e4m3"
                         else (int8, torch.int8, 4.0 / 127, 3.0 / 127))
    rng = np.random.default_rng(100 + G + D + bs)
    hkv = 2
    cache = PagedKVCache(3000, hkv, bs, D, dt, "cuda", rng.permutation(3000), fill=float("nan"), k_scale=ks,
                         v_scale=vs)
    g = torch.Generator().manual_seed(G + D)
    ids, hist = [], {}
    for fam in range(4):
        root = fam * 100
        n0 = int(rng.integers(64, 700))
        k0, v0 = torch.randn(n0, hkv, D, generator=g).bfloat16(), torch.randn(n0, hkv, D, generator=g).bfloat16()
        cache.add_sequence(root, k0.cuda(), v0.cuda())
        ids.append(root)
        hist[root] = ([k0], [v0])
        for j in range(1, int(rng.integers(1, 64 // G + 2))):
            cache.fork(root, root + j)
            ids.append(root + j)
            hist[root + j] = ([k0], [v0])
    for _ in range(int(rng.integers(1, 30))):       # private suffixes
        k = torch.randn(len(ids), hkv, D, generator=g).bfloat16()
        v = torch.randn(len(ids), hkv, D, generator=g).bfloat16()
        cache.append(ids, k.cuda(), v.cuda())
        for i, s in enumerate(ids):
            hist[s] = (hist[s][0] + [k[i:i + 1]], hist[s][1] + [v[i:i + 1]])
    q = torch.randn(len(ids), hkv * G, D, generator=g).bfloat16()
    a = cache.decode(ids, q.cuda(), D ** -0.5).cpu()
    b = cache.decode_cascade(ids, q.cuda(), D ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    assert len(cache.shared_prefix_groups(ids, 64 // G)[2]) > 0   # some prefix is shared
    assert float((a - b).abs().max()) <= 2e-3
    for i in (0, len(ids) // 2, len(ids) - 1):
        s = ids[i]
        K = codec.dequantize(codec.quantize(torch.cat(hist[s][0]).float().numpy(), ks), ks)
        V = codec.dequantize(codec.quantize(torch.cat(hist[s][1]).float().numpy(), vs), vs)
        ref = decode_attention(q[i], K, V, D ** -0.5)
        assert float(np.abs(b[i].double().numpy() - ref).max()) <= 4e-3


def test_llama2_7b_mha_fp8_cache():
    """The metric workload over an e4m3 cache: every sequence's codes equal the
    oracle's quantisation of its rows bitwise; every output row within the bf16
    bound of the fp64 attention over the dequantised rows."""
    from tests.parity import CodedReplay
    w = W.llama2_7b_mha()
    r = CodedReplay(w.shape, w.num_blocks, w.free_order, w.scale).run(W.simple_ops(w))
    r.check_pool_codes()
    r.check_outputs()


def test_llama2_7b_mha_int8_cache():
    """The metric workload over an int8 cache (scales 4/127, 3/127): codes equal
    the oracle's quantisation bitwise; every output row within the bf16 bound
    of the fp64 attention over the dequantised rows."""
    from tests.parity import CodedReplay
    w = W.llama2_7b_mha()
    r = CodedReplay(w.shape, w.num_blocks, w.free_order, w.scale, k_scale=4.0 / 127, v_scale=3.0 / 127,
                    fmt="int8").run(W.simple_ops(w))
    r.check_pool_codes()
    r.check_outputs()


def test_prefill_benchmark_size_sampled_rows():
    """The prefill benchmark's launch (8 prompts x 2048 tokens, 32/32 heads, D 128,
    bs 16, whole prompts in one pa_prefill): 24 sampled token rows of every
    prompt (first, last and across the 128-row tiles), all heads."""
    import torch
    from oracle.attention import decode_attention
    from paged_kv_cache_361_b200 import PagedKVCache
    nseq, plen, H, D, bs = 8, 2048, 32, 128, 16
    nb = nseq * plen // bs + 16
    cache = PagedKVCache(nb, H, bs, D, torch.bfloat16, "cuda", np.random.default_rng(3).permutation(nb),
                         fill=float("nan"))
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    T = nseq * plen
    q = torch.randn(T, H, D, generator=g, device="cuda").bfloat16()
    k = torch.randn(T, H, D, generator=g, device="cuda").bfloat16()
    v = torch.randn(T, H, D, generator=g, device="cuda").bfloat16()
    out = cache.prefill(list(range(nseq)), [plen] * nseq, q, k, v, D ** -0.5)
    assert B.pa_get_device_error()[0] == B.PA_OK
    rows = np.unique(np.r_[0, 1, 127, 128, 255, 256, 1000, 1023, 1024, 2047,
                           np.random.default_rng(5).integers(0, plen, 14)])
    worst = 0.0
    for s in range(nseq):
        base = s * plen
        K = k[base:base + plen].cpu()
        V = v[base:base + plen].cpu()
        for t in rows:
            ref = decode_attention(q[base + t].cpu(), K[:t + 1], V[:t + 1], D ** -0.5)
            err = float(np.abs(out[base + t].double().cpu().numpy() - ref).max())
            worst = max(worst, err)
    assert worst <= 4e-3, worst


def test_cascade_empty_suffix_and_empty_sequence():
    """A member whose whole context is the shared prefix (its suffix is empty)
    and an empty sequence: the suffix CTAs merge the prefix partials alone and
    write a zero row, as pa_decode does."""
    from paged_kv_cache_361_b200 import PagedKVCache
    hkv, G, D, bs = 2, 4, 128, 16
    g = torch.Generator().manual_seed(21)
    cache = PagedKVCache(64, hkv, bs, D, torch.bfloat16, "cuda", fill=float("nan"))
    k = torch.randn(128, hkv, D, generator=g).bfloat16()
    v = torch.randn(128, hkv, D, generator=g).bfloat16()
    cache.add_sequence(0, k.cuda(), v.cuda())          # 8 whole blocks: the prefix is all 128 tokens
    for child in (1, 2, 3):
        cache.fork(0, child)
    for _ in range(5):
        cache.append([1, 2], torch.randn(2, hkv, D, generator=g).bfloat16().cuda(),
                     torch.randn(2, hkv, D, generator=g).bfloat16().cuda())
    cache.add_sequence(9, torch.empty(0, hkv, D, dtype=torch.bfloat16).cuda(),
                       torch.empty(0, hkv, D, dtype=torch.bfloat16).cuda())
    ids = [0, 1, 2, 3, 9]
    off, mem, pre, sp, mp = cache.shared_prefix_groups(ids, 64 // G)
    assert pre.tolist() == [128] and sp.tolist() == [128, 128, 128, 128, 0]
    q = torch.randn(len(ids), hkv * G, D, generator=g).bfloat16().cuda()
    a = cache.decode(ids, q, D ** -0.5)
    b = cache.decode_cascade(ids, q, D ** -0.5)
    assert B.pa_get_device_error()[0] == B.PA_OK
    assert torch.isfinite(b).all()
    assert float(b[4].abs().max()) == 0.0
    assert float((a - b).abs().max()) <= 2e-3


def test_cascade_dispatch_order():
    """The suffix CTAs' dispatch order (seq_order) changes no result: no order,
    longest first and reversed give bitwise-equal outputs; an entry out of range
    is recorded as a bounds error and its row served in batch order."""
    from paged_kv_cache_361_b200 import PagedKVCache
    rng = np.random.default_rng(7)
    hkv, G, D, bs = 2, 4, 128, 16
    cache = PagedKVCache(4000, hkv, bs, D, torch.bfloat16, "cuda", rng.permutation(4000), fill=float("nan"))
    g = torch.Generator().manual_seed(7)
    ids = []
    for fam in range(4):
        root = fam * 100
        n0 = int(rng.integers(64, 600))
        cache.add_sequence(root, torch.randn(n0, hkv, D, generator=g).bfloat16().cuda(),
                           torch.randn(n0, hkv, D, generator=g).bfloat16().cuda())
        ids.append(root)
        for j in range(1, 6):
            cache.fork(root, root + j)
            ids.append(root + j)
    for s in ids:                                    # suffixes of different lengths
        for _ in range(int(rng.integers(0, 90))):
            cache.append([s], torch.randn(1, hkv, D, generator=g).bfloat16().cuda(),
                         torch.randn(1, hkv, D, generator=g).bfloat16().cuda())
    n = len(ids)
    q = torch.randn(n, hkv * G, D, generator=g).bfloat16().cuda()
    tables, lens, max_len = cache.decode_inputs(ids)
    offs, members, prefix, seq_prefix, max_pre = cache.shared_prefix_groups(ids, 64 // G)
    order = cache.bm.longest_first(ids, seq_prefix)
    span = np.array([cache.lens[s] for s in ids]) - seq_prefix
    assert sorted(order.tolist()) == list(range(n)) and (np.diff(span[order]) <= 0).all()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    ws = torch.empty(B.pa_decode_cascade_workspace_bytes(n, hkv * G, hkv, D, max_len, bs, max_pre),
                     dtype=torch.uint8, device="cuda")
    args = (t(offs), t(members), t(prefix), t(seq_prefix), int(max(np.diff(offs), default=0)), max_pre, ws)
    outs = []
    bad = np.arange(n, dtype=np.int32)
    bad[3] = n + 5
    for so in (None, order, order[::-1], bad):
        out = torch.full((n, hkv * G, D), float("nan"), dtype=torch.float32, device="cuda")
        B.pa_decode_cascade(q, cache.k_cache, cache.v_cache, t(tables), t(lens), D ** -0.5, out, max_len, *args,
                            seq_order=None if so is None else t(so))
        st, info = B.pa_get_device_error()
        assert (st, info) == ((B.PA_ERR_DEVICE_BOUNDS, n + 5) if so is bad else (B.PA_OK, 0))
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    ref = cache.decode(ids, q, D ** -0.5)
    assert float((ref - outs[0]).abs().max()) <= 2e-3


@pytest.mark.parametrize("dtype,G,part", [("bf16", 1, 0), ("bf16", 4, 0), ("bf16", 4, 128), ("bf16", 8, 256),
                                           ("bf16", 2, 64), ("e4m3", 1, 0), ("e4m3", 4, 128), ("int8", 8, 0)])
def test_decode_ordered_matches_decode(dtype, G, part):
    """pa_decode_ordered is pa_decode bit for bit whatever the order (longest
    first, reversed), on every kernel family: CUDA-core (G 1-2), tensor-core
    one-CTA-per-item and persistent (split), 8-bit; an out-of-range entry is
    recorded and its row served in batch order."""
    from paged_kv_cache_361_b200 import PagedKVCache
    rng = np.random.default_rng(G * 7 + part)
    hkv, D, bs = 2, 128, 16
    tdt = {"bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn, "int8": torch.int8}[dtype]
    sc = 4.0 / 127 if dtype == "int8" else 1.0
    cache = PagedKVCache(3000, hkv, bs, D, tdt, "cuda", rng.permutation(3000), k_scale=sc, v_scale=sc)
    g = torch.Generator().manual_seed(G + part)
    ids = list(range(23))
    for s in ids:
        n = int(rng.integers(1, 900))
        cache.add_sequence(s, torch.randn(n, hkv, D, generator=g).bfloat16().cuda(),
                           torch.randn(n, hkv, D, generator=g).bfloat16().cuda())
    n = len(ids)
    q = torch.randn(n, hkv * G, D, generator=g).bfloat16().cuda()
    tables, lens, max_len = cache.decode_inputs(ids)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    ws = torch.empty(max(256, B.pa_decode_workspace_bytes(n, hkv * G, hkv, D, max_len, bs, part)),
                     dtype=torch.uint8, device="cuda")
    order = cache.bm.longest_first(ids)
    assert (np.diff(lens[order]) <= 0).all()
    bad = np.arange(n, dtype=np.int32)
    bad[5] = -3
    outs = []
    for so in (None, order, order[::-1], bad):
        out = torch.full((n, hkv * G, D), float("nan"), dtype=torch.float32, device="cuda")
        B.pa_decode(q, cache.k_cache, cache.v_cache, t(tables), t(lens), D ** -0.5, out, max_len, part, ws,
                    seq_order=None if so is None else t(so))
        st, info = B.pa_get_device_error()
        assert (st, info) == ((B.PA_ERR_DEVICE_BOUNDS, -3) if so is bad else (B.PA_OK, 0))
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert torch.isfinite(outs[0]).all()


@pytest.mark.parametrize("dtype,G,part,bs", [("bf16", 1, 0, 16), ("bf16", 4, 0, 16), ("bf16", 4, 128, 16),
                                              ("bf16", 8, 256, 32), ("bf16", 2, 64, 8), ("e4m3", 1, 0, 16),
                                              ("e4m3", 4, 128, 16), ("int8", 8, 0, 16), ("int8", 2, 0, 4),
                                              ("fp32", 1, 0, 16), ("fp32", 4, 96, 16)])
def test_decode_append_matches_append_then_decode(dtype, G, part, bs):
    """pa_decode_append (the KV append done by the decode CTAs) leaves the same
    pool bytes and the same outputs, bit for bit, as pa_reshape_and_cache then
    pa_decode, on every kernel family; slot -1 writes nothing; a slot outside
    the pool is recorded and not written."""
    from paged_kv_cache_361_b200 import PagedKVCache
    rng = np.random.default_rng(G * 11 + part + bs)
    hkv, D = 2, 128
    tdt = {"bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn, "int8": torch.int8, "fp32": torch.float32}[dtype]
    idt = torch.float32 if dtype == "fp32" else torch.bfloat16
    sc = 4.0 / 127 if dtype == "int8" else 1.0
    nb = 4000 * 16 // bs
    cache = PagedKVCache(nb, hkv, bs, D, tdt, "cuda", rng.permutation(nb), fill=0.0, k_scale=sc, v_scale=sc)
    g = torch.Generator().manual_seed(G + part + bs)
    ids = list(range(19))
    for s in ids:
        n = int(rng.integers(0, 700))
        cache.add_sequence(s, torch.randn(n, hkv, D, generator=g).to(idt).cuda(),
                           torch.randn(n, hkv, D, generator=g).to(idt).cuda())
    slots, pairs = cache.bm.append_slots(ids)
    assert len(pairs) == 0
    for s in ids:
        cache.lens[s] += 1
    n = len(ids)
    tables, lens, max_len = cache.decode_inputs(ids)
    q = torch.randn(n, hkv * G, D, generator=g).to(idt).cuda()
    kn = torch.randn(n, hkv, D, generator=g).to(idt).cuda()
    vn = torch.randn(n, hkv, D, generator=g).to(idt).cuda()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    ws = torch.empty(max(256, B.pa_decode_workspace_bytes(n, hkv * G, hkv, D, max_len, bs, part)),
                     dtype=torch.uint8, device="cuda")
    order = t(cache.bm.longest_first(ids))
    pools = (cache.k_cache.clone(), cache.v_cache.clone())
    sl = torch.from_numpy(slots).cuda()

    def run(fused, slot_t):
        kc, vc = pools[0].clone(), pools[1].clone()
        if dtype in ("e4m3", "int8"):
            B.set_kv_scales(kc, vc, sc, sc)
        out = torch.full((n, hkv * G, D), float("nan"), dtype=torch.float32, device="cuda")
        if fused:
            B.pa_decode_append(q, kn, vn, slot_t, kc, vc, t(tables), t(lens), D ** -0.5, out, max_len, part, ws,
                               seq_order=order)
        else:
            B.pa_reshape_and_cache(kn, vn, slot_t, kc, vc)
            B.pa_decode(q, kc, vc, t(tables), t(lens), D ** -0.5, out, max_len, part, ws, seq_order=order)
        return out, kc, vc

    ref = run(False, sl)
    assert B.pa_get_device_error()[0] == B.PA_OK
    got = run(True, sl)
    assert B.pa_get_device_error()[0] == B.PA_OK
    assert torch.equal(got[0], ref[0])
    for a_, b_ in zip(got[1:], ref[1:]):
        assert torch.equal(a_.view(torch.uint8), b_.view(torch.uint8))
    # slot -1 for sequence 3 writes nothing there (its row keeps the old bytes), others as before
    sl2 = sl.clone()
    sl2[3] = -1
    ref2 = run(False, sl2)
    got2 = run(True, sl2)
    assert torch.equal(got2[0], ref2[0]) and torch.equal(got2[1].view(torch.uint8), ref2[1].view(torch.uint8))
    assert B.pa_get_device_error()[0] == B.PA_OK
    # a slot outside the pool: recorded, nothing written for it
    sl3 = sl2.clone()
    sl3[3] = nb * bs + 5
    got3 = run(True, sl3)
    st, info = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_BOUNDS and info == nb * bs + 5
    assert torch.equal(got3[1].view(torch.uint8), ref2[1].view(torch.uint8))
