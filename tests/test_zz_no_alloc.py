"""pa_decode_static_workspace: decode for callers that may not allocate device
memory (a runtime that owns the whole device and hands a kernel only its
inputs and outputs, or a serving loop where cudaMalloc's possible device
synchronisation is not allowed). The work counters and split partials go to a
fixed array inside the library instead of a caller workspace.

Checked through the C ABI against pa_decode with an allocated workspace. Both
run the same kernels on the same inputs, so the outputs must be bitwise equal:
on two calls in a row with different queries and lengths (the array keeps the
previous call's contents, which must not leak into the next result), for an
unsplit decode, the library's own split choice and 512-token partitions, and
for a split whose partials fill the array to just under its size. A split just
over the size is refused. Runs last so that a failure here leaves every other
test already run; it builds its own inputs, so it also passes alone.
"""
import pytest
import torch

from paged_kv_cache_361_b200 import PagedKVCache, binding as B

pytestmark = pytest.mark.gpu

LIMIT = 16 << 20   # PA_STATIC_WORKSPACE_BYTES


def _cache_with(lens, seed, hkv=8, D=128, bs=16):
    g = torch.Generator().manual_seed(seed)
    nb = sum(-(-L // bs) for L in lens) + 8
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, "cuda", fill=float("nan"))
    for s, L in enumerate(lens):
        cache.add_sequence(s, torch.randn(L, hkv, D, generator=g).bfloat16().cuda(),
                           torch.randn(L, hkv, D, generator=g).bfloat16().cuda())
    return cache, g


def _inputs(cache, ids):
    tables, lens, max_len = cache.decode_inputs(ids)
    return torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), max_len


def _pa_decode(cache, q, t, L, max_len, P):
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    nbytes = B.pa_decode_workspace_bytes(q.shape[0], q.shape[1], cache.k_cache.shape[1], q.shape[2], max_len,
                                         cache.block_size, P)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    B.pa_decode(q, cache.k_cache, cache.v_cache, t, L, 128 ** -0.5, out, max_len, P, ws)
    return out


def _static(cache, q, t, L, max_len, P):
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    B.pa_decode_static_workspace(q, cache.k_cache, cache.v_cache, t, L, 128 ** -0.5, out, max_len, P)
    return out


@pytest.mark.parametrize("P", [0, -1, 512])
def test_static_workspace_equals_pa_decode_twice(P):
    g0 = torch.Generator().manual_seed(0)
    lens = torch.randint(600, 2049, (16,), generator=g0).tolist()
    cache, g = _cache_with(lens, 0)
    hq, D = 32, 128
    for call, ids in enumerate(([*range(16)], [3, 7, 1, 12, 0, 9])):
        q = torch.randn(len(ids), hq, D, generator=g).bfloat16().cuda()
        t, L, max_len = _inputs(cache, ids)
        ref = _pa_decode(cache, q, t, L, max_len, P)
        out = _static(cache, q, t, L, max_len, P)
        torch.cuda.synchronize()
        assert B.pa_get_device_error()[0] == B.PA_OK
        assert torch.equal(out, ref), f"P={P} call {call}: max-abs {float((out - ref).abs().max())}"


def test_static_workspace_just_under_and_over_its_size():
    # 16 sequences x 32 query heads, 32-token partitions: every partition slot of
    # the 16 rows costs 16 * 32 * (2 + 128) * 4 bytes (about 260 KiB), so a longest
    # context of 2000 tokens (63 partitions) fits just under 16 MiB and one of
    # 2040 tokens (64 partitions) does not.
    hq, D, P = 32, 128, 32
    lens = [2000] + [1000 + 61 * i for i in range(1, 16)]
    cache, g = _cache_with(lens, 1)
    ids = list(range(16))
    t, L, max_len = _inputs(cache, ids)
    need = B.pa_decode_workspace_bytes(16, hq, 8, D, max_len, 16, P)
    assert need <= LIMIT and LIMIT - need < 300 << 10, need
    for _ in range(2):
        q = torch.randn(16, hq, D, generator=g).bfloat16().cuda()
        ref = _pa_decode(cache, q, t, L, max_len, P)
        out = _static(cache, q, t, L, max_len, P)
        torch.cuda.synchronize()
        assert B.pa_get_device_error()[0] == B.PA_OK
        assert torch.equal(out, ref)

    big_lens = [2040] + lens[1:]
    cache2, g2 = _cache_with(big_lens, 2)
    t2, L2, max_len2 = _inputs(cache2, ids)
    need2 = B.pa_decode_workspace_bytes(16, hq, 8, D, max_len2, 16, P)
    assert LIMIT < need2 < LIMIT + (300 << 10), need2
    q = torch.randn(16, hq, D, generator=g2).bfloat16().cuda()
    out = torch.empty(16, hq, D, device="cuda")
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_decode_static_workspace(q, cache2.k_cache, cache2.v_cache, t2, L2, 0.1, out, max_len2, P)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_static_workspace_rejects_oversized_split():
    lens = [700, 900]
    cache, g = _cache_with(lens, 3)
    hq, D = 32, 128
    q = torch.randn(2, hq, D, generator=g).bfloat16().cuda()
    out = torch.empty(2, hq, D, device="cuda")
    L = torch.tensor(lens, dtype=torch.int32, device="cuda")
    # a claimed max length of 2^20 tokens in 16-token partitions needs far more
    # than the fixed array
    big = 1 << 20
    assert B.pa_decode_workspace_bytes(2, hq, 8, D, big, 16, 16) > LIMIT
    bigt = torch.zeros(2, big // 16, dtype=torch.int32, device="cuda")
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_decode_static_workspace(q, cache.k_cache, cache.v_cache, bigt, L, 0.1, out, big, 16)
    assert e.value.status == B.PA_ERR_INVALID_ARG
