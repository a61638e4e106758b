"""pa_decode_static_workspace: decode for callers that may not allocate device
memory (a runtime that owns the whole device and hands a kernel only its
inputs and outputs, or a serving loop where cudaMalloc's possible device
synchronisation is not allowed). The split partials go to a fixed array inside
the library instead of a caller workspace.

Checked through the C ABI against pa_decode with an allocated workspace, on two
calls in a row with different queries and lengths (the array keeps the previous
call's contents, which must not leak into the next result), within the bf16
tolerance of the other parity tests. Runs last so that a failure here leaves
every other test already run; it builds its own inputs, so it also passes alone.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_361_b200 import PagedKVCache, binding as B

pytestmark = pytest.mark.gpu

TOL = 4e-3   # bf16 cache, fp32 accumulation, as in the other parity tests


def _setup(seed):
    g = torch.Generator().manual_seed(seed)
    nseq, hq, hkv, D, bs = 16, 32, 8, 128, 16
    lens = torch.randint(600, 2049, (nseq,), generator=g).tolist()
    nb = sum(-(-L // bs) for L in lens) + 8
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, "cuda", fill=float("nan"))
    for s, L in enumerate(lens):
        k = torch.randn(L, hkv, D, generator=g).bfloat16().cuda()
        v = torch.randn(L, hkv, D, generator=g).bfloat16().cuda()
        cache.add_sequence(s, k, v)
    return cache, lens, g, hq, D


def _reference(cache, ids, q, P):
    tables, lens, max_len = cache.decode_inputs(ids)
    t = torch.from_numpy(tables).cuda()
    L = torch.from_numpy(lens).cuda()
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    nbytes = B.pa_decode_workspace_bytes(len(ids), q.shape[1], cache.k_cache.shape[1], q.shape[2], max_len,
                                         cache.block_size, P)
    assert nbytes > 0   # the split is used, so the workspace matters
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    B.pa_decode(q, cache.k_cache, cache.v_cache, t, L, 128 ** -0.5, out, max_len, P, ws)
    return out, t, L, max_len


def test_static_workspace_matches_pa_decode_twice():
    cache, lens, g, hq, D = _setup(0)
    P = 512
    for call, ids in enumerate(([*range(16)], [3, 7, 1, 12, 0, 9])):
        q = torch.randn(len(ids), hq, D, generator=g).bfloat16().cuda()
        ref, t, L, max_len = _reference(cache, ids, q, P)
        out = torch.full_like(ref, float("nan"))
        B.pa_decode_static_workspace(q, cache.k_cache, cache.v_cache, t, L, 128 ** -0.5, out, max_len, P)
        torch.cuda.synchronize()
        assert B.pa_get_device_error()[0] == B.PA_OK
        err = float((out - ref).abs().max())
        assert np.isfinite(err) and err <= TOL, f"call {call}: max-abs {err}"


def test_static_workspace_rejects_oversized_split():
    cache, lens, g, hq, D = _setup(1)
    ids = [0, 1]
    q = torch.randn(2, hq, D, generator=g).bfloat16().cuda()
    tables, lens_np, max_len = cache.decode_inputs(ids)
    t = torch.from_numpy(tables).cuda()
    L = torch.from_numpy(lens_np).cuda()
    out = torch.empty(2, hq, D, device="cuda")
    # 16-token partitions over 2 x 32 heads x ~128 parts x 130 floats would fit; a
    # claimed max length of 2^20 tokens needs far more than the fixed array
    big = 1 << 20
    assert B.pa_decode_workspace_bytes(2, hq, 8, D, big, 16, 16) > (16 << 20)
    bigt = torch.zeros(2, big // 16, dtype=torch.int32, device="cuda")
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_decode_static_workspace(q, cache.k_cache, cache.v_cache, bigt, L, 0.1, out, big, 16)
    assert e.value.status == B.PA_ERR_INVALID_ARG
