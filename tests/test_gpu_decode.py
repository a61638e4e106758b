"""GPU parity of pa_decode / pa_reshape_and_cache / pa_copy_blocks against the
oracle on small seeded cases: every block size, head size, group size and
dtype, split and unsplit, plus the degenerate and error cases."""
import math
import zlib

import numpy as np
import pytest
import torch

from paged_kv_cache_361_b200 import PagedKVCache, binding as B
from paged_kv_cache_361_b200 import workloads as W
from tests.parity import Replay, TOL, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    if torch.cuda.is_available():
        B.pa_get_device_error()
    yield


def test_tiny_fp32_config():
    """2 sequences of 10 and 7 tokens (the first is the pages' 10-token example),
    4 heads, head_dim 64, block_size 4, pool 16: full pool and outputs."""
    w = W.tiny_fp32()
    r = Replay(w.shape, w.num_blocks, w.free_order, w.scale).run(W.simple_ops(w))
    r.check_pool_bitwise()
    err = r.check_outputs(tol=1e-5)
    assert err <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 32])
def test_fuzz_shapes(dtype, D, G, bs):
    hkv = 2
    sh = W.Shape(hkv * G, hkv, D, bs, dtype)
    seed = zlib.crc32(f"{dtype}-{D}-{G}-{bs}".encode()) % 100000
    w = W.random_small(seed, num_seqs=6, shape=sh, max_len=int(np.random.default_rng(seed).integers(40, 300)))
    for P in (0, -1, max(bs, 32), 2 * bs):
        r = Replay(sh, w.num_blocks, w.free_order, w.scale, partition_tokens=P).run(W.simple_ops(w))
        r.check_outputs()
    r.check_pool_bitwise()


@pytest.mark.parametrize("P", [0, 16, 48, 64, 512, -1])
def test_partitions_agree(P):
    """Splitting a sequence into partitions and merging equals the oracle."""
    sh = W.Shape(8, 2, 128, 16, "bf16")
    w = W.random_small(11, num_seqs=5, shape=sh, max_len=1500)
    r = Replay(sh, w.num_blocks, w.free_order, w.scale, partition_tokens=P).run(W.simple_ops(w))
    r.check_outputs()


def test_empty_context_gives_zero_rows():
    sh = W.Shape(4, 2, 64, 8, "bf16")
    cache = PagedKVCache(8, 2, 8, 64, torch.bfloat16, "cuda", fill=float("nan"))
    cache.add_sequence(0, torch.zeros(0, 2, 64, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(0, 2, 64, dtype=torch.bfloat16, device="cuda"))
    k = torch.randn(5, 2, 64, device="cuda").bfloat16()
    cache.add_sequence(1, k, k)
    q = torch.randn(2, 4, 64, device="cuda").bfloat16()
    for P in (0, 8, -1):
        out = cache.decode([0, 1], q, 0.125, partition_tokens=P)
        assert torch.equal(out[0], torch.zeros_like(out[0]))
        assert torch.isfinite(out[1]).all()
    assert B.pa_get_device_error()[0] == B.PA_OK


def test_single_token_context_returns_v():
    sh = W.Shape(8, 1, 128, 16, "bf16")
    cache = PagedKVCache(4, 1, 16, 128, torch.bfloat16, "cuda", fill=float("nan"))
    k = torch.randn(1, 1, 128, device="cuda").bfloat16()
    v = torch.randn(1, 1, 128, device="cuda").bfloat16()
    cache.add_sequence(7, k, v)
    out = cache.decode([7], torch.randn(1, 8, 128, device="cuda").bfloat16(), 0.1)
    assert torch.equal(out[0], v[0, 0].float().expand(8, 128))


def test_physical_permutation_is_bitwise_invisible():
    """Same sequences, different physical placement: identical output bits."""
    sh = W.Shape(16, 4, 128, 16, "bf16")
    w = W.random_small(5, num_seqs=4, shape=sh, max_len=700)
    outs = []
    for perm in range(3):
        order = np.random.default_rng(perm).permutation(w.num_blocks)
        r = Replay(sh, w.num_blocks, order, w.scale).run(W.simple_ops(w))
        outs.append(r.decodes[-1][2])
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_copy_blocks_bitwise_and_bounds():
    kc = torch.randn(10, 4, 16, 128, device="cuda").bfloat16()
    vc = torch.randn(10, 4, 16, 128, device="cuda").bfloat16()
    k0, v0 = kc.clone(), vc.clone()
    pairs = torch.tensor([[1, 7], [2, 8], [3, 9]], dtype=torch.int32, device="cuda")
    B.pa_copy_blocks(kc, vc, pairs)
    for s_, d_ in [(1, 7), (2, 8), (3, 9)]:
        assert torch.equal(bits(kc[d_]), bits(k0[s_])) and torch.equal(bits(vc[d_]), bits(v0[s_]))
    for b in range(7):
        assert torch.equal(bits(kc[b]), bits(k0[b]))
    assert B.pa_get_device_error()[0] == B.PA_OK
    bad = torch.tensor([[0, 10]], dtype=torch.int32, device="cuda")
    B.pa_copy_blocks(kc, vc, bad)
    st, info = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_BOUNDS and info == 10


def test_reshape_and_cache_skip_and_bounds():
    kc = torch.zeros(4, 2, 4, 64, device="cuda")
    vc = torch.zeros(4, 2, 4, 64, device="cuda")
    k = torch.randn(3, 2, 64, device="cuda")
    v = torch.randn(3, 2, 64, device="cuda")
    B.pa_reshape_and_cache(k, v, torch.tensor([5, -1, 15], device="cuda"), kc, vc)
    assert torch.equal(kc[1, :, 1], k[0]) and torch.equal(vc[3, :, 3], v[2])
    assert int((kc != 0).sum()) == 2 * 2 * 64
    assert B.pa_get_device_error()[0] == B.PA_OK
    B.pa_reshape_and_cache(k, v, torch.tensor([0, 16, -2], device="cuda"), kc, vc)
    st, info = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_BOUNDS and info in (16, -2)


def test_decode_bad_block_id_and_length_are_reported():
    cache = PagedKVCache(4, 1, 16, 64, torch.bfloat16, "cuda", fill=0.0)
    q = torch.randn(1, 1, 64, device="cuda").bfloat16()
    out = torch.empty(1, 1, 64, device="cuda")
    tables = torch.tensor([[0, 9]], dtype=torch.int32, device="cuda")
    ws = torch.empty(B.pa_decode_workspace_bytes(1, 1, 1, 64, 32, 16, 0), dtype=torch.uint8, device="cuda")
    B.pa_decode(q, cache.k_cache, cache.v_cache, tables, torch.tensor([20], dtype=torch.int32, device="cuda"),
                0.1, out, 32, 0, ws)
    st, info = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_BOUNDS and info == 9
    B.pa_decode(q, cache.k_cache, cache.v_cache, tables, torch.tensor([40], dtype=torch.int32, device="cuda"),
                0.1, out, 32, 0, ws)
    st, info = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_BOUNDS and info == 40


def test_wait_limit_returns_status():
    """A wait that nothing completes ends with PA_ERR_DEVICE_TIMEOUT; the context stays usable."""
    B.pa_selftest_wait_timeout(50_000_000)
    st, _ = B.pa_get_device_error()
    assert st == B.PA_ERR_DEVICE_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


def test_step_host_matches_oracle_with_cow():
    """pa_step_host (host buffers in, host buffer out) on a prefix-sharing batch:
    the first step copies the shared partial block; slots, pairs and outputs match
    the oracle."""
    from oracle.replay import OracleRun
    sh = W.Shape(16, 4, 128, 16, "bf16")
    g = torch.Generator().manual_seed(3)
    ref = OracleRun(sh, 64, list(range(64)), keep_pool=True)
    cache = PagedKVCache(64, 4, 16, 128, torch.bfloat16, "cuda", list(range(64)), fill=float("nan"))
    pk, pv = torch.randn(37, 4, 128, generator=g).bfloat16(), torch.randn(37, 4, 128, generator=g).bfloat16()
    add = ("add", 0, 37, lambda which, device="cpu": pk if which == "k" else pv)
    ref.apply(add)
    cache.add_sequence(0, pk.cuda(), pv.cuda())
    for child in (1, 2):
        ref.apply(("fork", 0, child))
        cache.fork(0, child)
    ids = [2, 0, 1]
    for step in range(3):
        q = torch.randn(3, 16, 128, generator=g).bfloat16().pin_memory()
        k = torch.randn(3, 4, 128, generator=g).bfloat16().pin_memory()
        v = torch.randn(3, 4, 128, generator=g).bfloat16().pin_memory()
        out = torch.empty(3, 16, 128, dtype=torch.float32).pin_memory()
        rec = ref.apply(("append", ids, lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
        cache.step_host(ids, q, k, v, out, 128 ** -0.5, partition_tokens=16 if step == 1 else -1)
        if step == 0:
            assert len(rec["pairs"]) == 2
        for i, s in enumerate(ids):
            exp = ref.attend(s, q[i], 128 ** -0.5, use_pool=True)
            assert float(np.abs(out[i].double().numpy() - exp).max()) <= TOL["bf16"]
    assert B.pa_get_device_error()[0] == B.PA_OK
    for s in ids:
        assert cache.bm.block_table(s)[0].tolist() == ref.bm.block_table(s)


def test_step_host_rejects_small_staging_without_change():
    cache = PagedKVCache(8, 1, 16, 64, torch.bfloat16, "cuda")
    cache.add_sequence(0, torch.zeros(3, 1, 64, dtype=torch.bfloat16, device="cuda"),
                       torch.zeros(3, 1, 64, dtype=torch.bfloat16, device="cuda"))
    q = torch.zeros(1, 1, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 64, dtype=torch.bfloat16)
    out = torch.empty(1, 1, 64)
    tiny_dev = torch.empty(256, dtype=torch.uint8, device="cuda")
    tiny_host = torch.empty(256, dtype=torch.uint8)
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_step_host(cache.bm, cache.k_cache, cache.v_cache, [0], q, k, k, 0.1, out, tiny_dev, tiny_host)
    assert e.value.status == B.PA_ERR_INVALID_ARG
    assert cache.bm.block_table(0)[1] == 3


def test_swap_out_reuse_swap_in_decode():
    """P2 §五: a sequence's blocks move to a pinned host pool, other sequences
    reuse the released device blocks, the sequence comes back into fresh blocks
    and decodes exactly as before."""
    from oracle.replay import OracleRun
    g = torch.Generator().manual_seed(5)
    sh = W.Shape(8, 2, 128, 16, "bf16")
    cache = PagedKVCache(12, 2, 16, 128, torch.bfloat16, "cuda", list(range(12)), fill=float("nan"))
    cache.enable_swap(16)
    rows = {s: (torch.randn(70, 2, 128, generator=g).bfloat16(), torch.randn(70, 2, 128, generator=g).bfloat16())
            for s in (1, 2)}
    for s in (1, 2):
        cache.add_sequence(s, rows[s][0][:40].cuda(), rows[s][1][:40].cuda())
    dev_blocks = cache.bm.block_table(1)[0].tolist()
    before = cache.k_cache[dev_blocks].cpu()
    pairs = cache.swap_out(1)
    assert pairs[:, 0].tolist() == dev_blocks
    torch.cuda.synchronize()
    assert torch.equal(bits(cache.host_k[pairs[:, 1].tolist()]), bits(before))
    # sequence 3 takes every free block, the released ones included, and overwrites them
    junk = torch.randn(144, 2, 128, generator=g).bfloat16()
    cache.add_sequence(3, junk.cuda(), junk.cuda())
    assert set(cache.bm.block_table(3)[0].tolist()) & set(dev_blocks)
    cache.free(2)
    back = cache.swap_in(1)
    assert back[:, 0].tolist() == pairs[:, 1].tolist()
    q = torch.randn(1, 8, 128, generator=g).bfloat16()
    out = cache.decode([1], q.cuda(), 128 ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    from oracle.attention import decode_attention
    ref = decode_attention(q[0], rows[1][0][:40], rows[1][1][:40], 128 ** -0.5)
    assert float(np.abs(out[0].double().numpy() - ref).max()) <= TOL["bf16"]


def test_swap_blocks_rejects_pageable_host_memory():
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    hk = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16)      # pageable
    pairs = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_swap_blocks(kc, kc, hk, hk, pairs, True)
    assert e.value.status == B.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_prefill_chunked_matches_oracle(G, D, bs):
    """Chunked prefill: existing sequences grow by a chunk, new ones start; every
    new token's causal attention over the paged cache matches the oracle."""
    from oracle.prefill import prefill_attention
    rng = np.random.default_rng(G * 1000 + D + bs)
    hkv = 2
    nseq = 5
    pre = rng.integers(0, 300, size=nseq)
    pre[0] = 0
    chunk = rng.integers(1, 200, size=nseq)
    chunk[1] = 128 // G           # exactly one 128-row query tile
    chunk[2] = 64 // G            # half a tile
    nb = int(sum(-(-int(p + c) // bs) for p, c in zip(pre, chunk))) + 4
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, "cuda", rng.permutation(nb), fill=float("nan"))
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    K = {s: torch.randn(int(pre[s] + chunk[s]), hkv, D, generator=g).bfloat16() for s in range(nseq)}
    V = {s: torch.randn(int(pre[s] + chunk[s]), hkv, D, generator=g).bfloat16() for s in range(nseq)}
    for s in range(nseq):
        if pre[s]:
            cache.add_sequence(s, K[s][:pre[s]].cuda(), V[s][:pre[s]].cuda())
    q = torch.randn(int(chunk.sum()), hkv * G, D, generator=g).bfloat16()
    k_new = torch.cat([K[s][pre[s]:] for s in range(nseq)])
    v_new = torch.cat([V[s][pre[s]:] for s in range(nseq)])
    out = cache.prefill(list(range(nseq)), chunk, q.cuda(), k_new.cuda(), v_new.cuda(), D ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    row = 0
    for s in range(nseq):
        n = int(chunk[s])
        ref = prefill_attention(q[row:row + n], K[s], V[s], D ** -0.5)
        err = float(np.abs(out[row:row + n].double().numpy() - ref).max())
        assert err <= TOL["bf16"], f"seq {s}: {err}"
        row += n


@pytest.mark.parametrize("G,D", [(1, 128), (8, 128), (4, 64)])
def test_prefill_long_chunk_many_tiles(G, D):
    """A 700-token chunk after 900 cached tokens: many query tiles and 25 key
    chunks, a ragged last tile and last key chunk, NaN padding in the pool."""
    from oracle.prefill import prefill_attention
    hkv, bs = 2, 16
    g = torch.Generator().manual_seed(40 + G + D)
    pre, n = 900, 700
    nb = -(-(pre + n) // bs) + 3
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, "cuda", np.random.default_rng(G).permutation(nb),
                         fill=float("nan"))
    K = torch.randn(pre + n, hkv, D, generator=g).bfloat16()
    V = torch.randn(pre + n, hkv, D, generator=g).bfloat16()
    cache.add_sequence(0, K[:pre].cuda(), V[:pre].cuda())
    q = torch.randn(n, hkv * G, D, generator=g).bfloat16()
    out = cache.prefill([0], [n], q.cuda(), K[pre:].cuda(), V[pre:].cuda(), D ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    rows = np.r_[0:40, 300:340, n - 40:n]
    ref = prefill_attention(q, K, V, D ** -0.5)
    err = float(np.abs(out.double().numpy()[rows] - ref[rows]).max())
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("vscale", [2000.0, 1e-3])
def test_prefill_value_range_through_f16(vscale):
    """The prefill reads V as f16 (its P V product is f16 x f16): V rows scaled
    to |v| of a few thousand, or down to about 1e-3, come out within the bf16
    tolerance scaled by the same factor."""
    from oracle.prefill import prefill_attention
    hkv, bs, D, G = 2, 16, 128, 4
    g = torch.Generator().manual_seed(77)
    n = 300
    cache = PagedKVCache(-(-n // bs) + 2, hkv, bs, D, torch.bfloat16, "cuda", fill=float("nan"))
    K = torch.randn(n, hkv, D, generator=g).bfloat16()
    V = (torch.randn(n, hkv, D, generator=g) * vscale).bfloat16()
    q = torch.randn(n, hkv * G, D, generator=g).bfloat16()
    out = cache.prefill([0], [n], q.cuda(), K.cuda(), V.cuda(), D ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    ref = prefill_attention(q, K, V, D ** -0.5)
    err = float(np.abs(out.double().numpy() - ref).max())
    assert err <= TOL["bf16"] * vscale, err


def test_prefill_then_decode_consistent():
    """The last token of a whole-prompt prefill and a decode over the cache the
    prefill wrote both match the oracle's attention of that token over the
    whole prompt (the two kernels round differently, so they are compared with
    the oracle, not with each other)."""
    from oracle.attention import decode_attention
    cache = PagedKVCache(64, 4, 16, 128, torch.bfloat16, "cuda", fill=float("nan"))
    g = torch.Generator().manual_seed(9)
    k = torch.randn(300, 4, 128, generator=g).bfloat16()
    v = torch.randn(300, 4, 128, generator=g).bfloat16()
    q = torch.randn(300, 16, 128, generator=g).bfloat16()
    out = cache.prefill([7], [300], q.cuda(), k.cuda(), v.cuda(), 128 ** -0.5)
    dec = cache.decode([7], q[-1:].cuda(), 128 ** -0.5)
    assert B.pa_get_device_error()[0] == B.PA_OK
    ref = decode_attention(q[-1], k, v, 128 ** -0.5)
    assert float(np.abs(out[-1].cpu().double().numpy() - ref).max()) <= TOL["bf16"]
    assert float(np.abs(dec[0].cpu().double().numpy() - ref).max()) <= TOL["bf16"]


def test_step_plan_matches_oracle():
    """The prepared pa_step_host call (one native call per step) over three steps."""
    from oracle.replay import OracleRun
    g = torch.Generator().manual_seed(8)
    sh = W.Shape(4, 4, 64, 8, "bf16")
    ref = OracleRun(sh, 40, list(range(40)), keep_pool=True)
    cache = PagedKVCache(40, 4, 8, 64, torch.bfloat16, "cuda", list(range(40)), fill=float("nan"))
    for s, n in ((0, 13), (1, 30), (2, 1)):
        k, v = torch.randn(n, 4, 64, generator=g).bfloat16(), torch.randn(n, 4, 64, generator=g).bfloat16()
        ref.apply(("add", s, n, lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
        cache.add_sequence(s, k.cuda(), v.cuda())
    ids = [1, 0, 2]
    q = torch.empty(3, 4, 64, dtype=torch.bfloat16).pin_memory()
    k = torch.empty(3, 4, 64, dtype=torch.bfloat16).pin_memory()
    v = torch.empty(3, 4, 64, dtype=torch.bfloat16).pin_memory()
    out = torch.empty(3, 4, 64).pin_memory()
    plan = cache.step_plan(ids, q, k, v, out, 0.125, max_context_len=64)
    for step in range(3):
        q.copy_(torch.randn(3, 4, 64, generator=g).bfloat16())
        k.copy_(torch.randn(3, 4, 64, generator=g).bfloat16())
        v.copy_(torch.randn(3, 4, 64, generator=g).bfloat16())
        kk, vv = k.clone(), v.clone()
        ref.apply(("append", ids, lambda which, device="cpu": kk if which == "k" else vv))
        plan.run()
        for i, s in enumerate(ids):
            exp = ref.attend(s, q[i], 0.125, use_pool=True)
            assert float(np.abs(out[i].double().numpy() - exp).max()) <= TOL["bf16"]


def test_swap_copy_engine_equals_kernel_swap():
    """pa_swap_blocks_copy (copy engines, host pairs; runs of consecutive ids
    merged into one copy) moves the same bytes as the pa_swap_blocks kernel."""
    g = torch.Generator().manual_seed(9)
    kc = torch.randn(40, 2, 16, 64, generator=g).bfloat16().cuda()
    vc = torch.randn(40, 2, 16, 64, generator=g).bfloat16().cuda()
    shape = (24, 2, 16, 64)
    hk1, hv1 = (torch.zeros(shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2))
    hk2, hv2 = (torch.zeros(shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2))
    # scattered ids plus a run of five consecutive (device, host) pairs
    pairs = np.array([[7, 3], [30, 0], [11, 12], [12, 13], [13, 14], [14, 15], [15, 16], [2, 23], [39, 1]],
                     dtype=np.int32)
    B.pa_swap_blocks(kc, vc, hk1, hv1, torch.from_numpy(pairs).cuda(), True)
    B.pa_swap_blocks_copy(kc, vc, hk2, hv2, pairs, True)
    torch.cuda.synchronize()
    assert torch.equal(bits(hk1), bits(hk2)) and torch.equal(bits(hv1), bits(hv2))
    assert torch.equal(bits(hk2[pairs[:, 1]]), bits(kc[pairs[:, 0]].cpu()))
    # and back into other device blocks
    back = np.stack([pairs[:, 1], np.arange(20, 29, dtype=np.int32)], 1)
    kc2, vc2 = kc.clone(), vc.clone()
    B.pa_swap_blocks(kc, vc, hk1, hv1, torch.from_numpy(back).cuda(), False)
    B.pa_swap_blocks_copy(kc2, vc2, hk2, hv2, back, False)
    torch.cuda.synchronize()
    assert B.pa_get_device_error()[0] == B.PA_OK
    assert torch.equal(bits(kc), bits(kc2)) and torch.equal(bits(vc), bits(vc2))


def test_swap_copy_engine_checks_ids_on_the_host():
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    hk = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, pin_memory=True)
    for bad in ([[0, 4]], [[4, 0]], [[-1, 0]]):
        with pytest.raises(B.PagedAttnError) as e:
            B.pa_swap_blocks_copy(kc, kc, hk, hk, np.array(bad, np.int32), True)
        assert e.value.status == B.PA_ERR_INVALID_ARG
    pageable = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_swap_blocks_copy(kc, kc, pageable, pageable, np.array([[0, 1]], np.int32), True)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_step_host_phase_timers():
    g = torch.Generator().manual_seed(4)
    cache = PagedKVCache(64, 2, 16, 128, torch.bfloat16, "cuda")
    for s in range(3):
        cache.add_sequence(s, torch.randn(50, 2, 128, generator=g).bfloat16().cuda(),
                           torch.randn(50, 2, 128, generator=g).bfloat16().cuda())
    q = torch.randn(3, 8, 128, generator=g).bfloat16().pin_memory()
    k = torch.randn(3, 2, 128, generator=g).bfloat16().pin_memory()
    out = torch.empty(3, 8, 128, pin_memory=True)
    cache.step_host([0, 1, 2], q, k, k, out)
    t = B.pa_step_host_last_timing()
    parts = ("block_manager_us", "metadata_enqueue_us", "chains_enqueue_us", "wait_us")
    assert all(t[p] >= 0 for p in parts) and t["total_us"] > 0 and t["chunks"] == 1
    assert sum(t[p] for p in parts) <= t["total_us"] * 1.0001 + 1e-3


@pytest.mark.parametrize("dtype,G", [("f32", 1), ("bf16", 1), ("bf16", 4), ("bf16", 8)])
def test_last_cta_merge_and_merge_kernel_agree_with_oracle(dtype, G):
    """Few partitions (2..7) are merged by the last CTA of each (sequence, kv
    head); many by the merge kernel. Both against the oracle."""
    sh = W.Shape(2 * G, 2, 128, 16, dtype)
    w = W.random_small(31 + G, num_seqs=5, shape=sh, max_len=700)
    for P in (128, 16):   # <= 6 partitions of 128 tokens; up to 44 of 16
        r = Replay(sh, w.num_blocks, w.free_order, w.scale, partition_tokens=P).run(W.simple_ops(w))
        r.check_outputs()


@pytest.mark.parametrize("n,G", [(16, 4), (37, 1), (64, 8)])
def test_step_host_chunked_matches_oracle(n, G):
    """A batch of 16 or more sequences runs as row chunks on the library's own
    streams (copies of one chunk overlap another's kernels); families of forked
    sequences make the first step copy shared blocks. Slots, pairs, tables and
    every output row match the oracle over three steps, one of them split."""
    from oracle.replay import OracleRun
    hkv, D, bs = 2, 128, 16
    sh = W.Shape(hkv * G, hkv, D, bs, "bf16")
    rng = np.random.default_rng(n * 10 + G)
    nb = 24 * n
    order = rng.permutation(nb)
    ref = OracleRun(sh, nb, order, keep_pool=True)
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, "cuda", order, fill=float("nan"))
    g = torch.Generator().manual_seed(n + G)
    ids = []
    s = 0
    while len(ids) < n:
        L = int(rng.integers(1, 300))
        k = torch.randn(L, hkv, D, generator=g).bfloat16()
        v = torch.randn(L, hkv, D, generator=g).bfloat16()
        ref.apply(("add", s, L, lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
        cache.add_sequence(s, k.cuda(), v.cuda())
        ids.append(s)
        for j in range(int(rng.integers(0, 3))):   # forks share the prompt's blocks
            if len(ids) < n:
                ref.apply(("fork", s, s + 1 + j))
                cache.fork(s, s + 1 + j)
                ids.append(s + 1 + j)
        s += 10
    ids = [int(x) for x in rng.permutation(ids)]
    for step in range(3):
        q = torch.randn(n, hkv * G, D, generator=g).bfloat16().pin_memory()
        k = torch.randn(n, hkv, D, generator=g).bfloat16().pin_memory()
        v = torch.randn(n, hkv, D, generator=g).bfloat16().pin_memory()
        out = torch.full((n, hkv * G, D), float("nan"), dtype=torch.float32).pin_memory()
        ref.apply(("append", ids, lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
        cache.step_host(ids, q, k, v, out, D ** -0.5, partition_tokens=64 if step == 1 else -1)
        assert B.pa_step_host_last_timing()["chunks"] >= 2          # the chained path
        for i, sid in enumerate(ids):
            exp = ref.attend(sid, q[i], D ** -0.5, use_pool=True)
            assert float(np.abs(out[i].double().numpy() - exp).max()) <= TOL["bf16"], (step, sid)
    assert B.pa_get_device_error()[0] == B.PA_OK
    for sid in ids:
        assert cache.bm.block_table(sid)[0].tolist() == ref.bm.block_table(sid)
