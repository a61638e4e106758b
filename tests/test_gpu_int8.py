"""GPU parity of the int8 KV cache (symmetric codes in [-127, 127], per-tensor
K and V scales, bf16 inputs) against the oracle: the codes pa_reshape_and_cache
stores are compared bit for bit with oracle/int8.py's quantiser, and pa_decode
and pa_prefill with the fp64 attention over the oracle's dequantised rows.
Block copies and swaps move codes unchanged. Pool padding is -128, the code
quantisation never writes."""
import zlib

import numpy as np
import pytest
import torch

from oracle import int8
from oracle.attention import decode_attention
from oracle.replay import OracleRun
from paged_kv_cache_361_b200 import PagedKVCache, binding as B
from paged_kv_cache_361_b200 import workloads as W
from tests.parity import TOL, CodedReplay

pytestmark = pytest.mark.gpu

# Codes are integers times a scale and q is bf16: the bf16 bound applies.
TOL8 = TOL["bf16"]
# N(0, 1) rows: |x| up to 4 uses the whole code range; larger values clamp
K_SCALE, V_SCALE = 4.0 / 127.0, 3.0 / 127.0


@pytest.fixture(autouse=True)
def _clean_error_word():
    if torch.cuda.is_available():
        B.pa_get_device_error()
    yield


def _replay(sh, nb, order, scale, P=-1):
    return CodedReplay(sh, nb, order, scale, partition_tokens=P, k_scale=K_SCALE, v_scale=V_SCALE, fmt="int8")


def _dq(x, scale):
    return int8.dequantize(int8.quantize(x.float().numpy(), scale), scale)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_int8_fuzz_shapes(D, G, bs):
    hkv = 2
    sh = W.Shape(hkv * G, hkv, D, bs, "bf16")
    seed = zlib.crc32(f"int8-{D}-{G}-{bs}".encode()) % 100000
    w = W.random_small(seed, num_seqs=6, shape=sh, max_len=int(np.random.default_rng(seed).integers(40, 400)))
    for P in (0, -1, 2 * max(bs, 16)):
        r = _replay(sh, w.num_blocks, w.free_order, w.scale, P).run(W.simple_ops(w))
        r.check_outputs(tol=TOL8)
    r.check_pool_codes()


def test_int8_long_split_and_mha():
    """Llama-2-7B-shaped heads (32 x 128, MHA), a 4k-token sequence cut into partitions."""
    sh = W.Shape(32, 32, 128, 16, "bf16")
    w = W.random_small(22, num_seqs=3, shape=sh, max_len=4096)
    for P in (0, 512, -1):
        r = _replay(sh, w.num_blocks, w.free_order, w.scale, P).run(W.simple_ops(w))
        r.check_outputs(tol=TOL8)
    r.check_pool_codes()


def test_int8_fork_copy_on_write():
    sh = W.Shape(8, 2, 128, 16, "bf16")
    g = torch.Generator().manual_seed(18)
    pk, pv = torch.randn(37, 2, 128, generator=g).bfloat16(), torch.randn(37, 2, 128, generator=g).bfloat16()
    ops = [("add", 0, 37, lambda which, device="cpu": pk if which == "k" else pv),
           ("fork", 0, 1), ("fork", 0, 2)]
    for step in range(5):
        k, v = torch.randn(3, 2, 128, generator=g).bfloat16(), torch.randn(3, 2, 128, generator=g).bfloat16()
        ops.append(("append", [2, 0, 1], lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
    q = torch.randn(3, 8, 128, generator=g).bfloat16()
    ops.append(("decode", [0, 1, 2], lambda device="cpu": q))
    r = _replay(sh, 20, list(range(20)), 128 ** -0.5).run(ops)
    assert r.n_pairs == 2
    r.check_pool_codes()
    r.check_outputs(tol=TOL8)


def test_int8_reshape_clamps_ties_and_nan():
    """Values past the range clamp to +-127; ties round to even; NaN becomes 0;
    the codes equal the oracle's bit for bit."""
    hkv, D, bs = 2, 64, 8
    cache = PagedKVCache(4, hkv, bs, D, torch.int8, "cuda", list(range(4)), fill=float("nan"), k_scale=0.5,
                         v_scale=0.25)
    g = torch.Generator().manual_seed(14)
    k = (torch.randn(11, hkv, D, generator=g) * 100).bfloat16()
    v = (torch.randn(11, hkv, D, generator=g) * 10).bfloat16()
    k[0, 0, :8] = torch.tensor([float("inf"), -float("inf"), 1e30, -1e30, float("nan"), 0.25, 0.75, -1.25])
    v[3, 1, :4] = torch.tensor([31.875, 31.625, -32.0, 0.125])   # 127.5 -> 127, 126.5 -> 126, -128 -> -127, 0.5 -> 0
    cache.add_sequence(0, k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert B.pa_get_device_error()[0] == B.PA_OK
    t = torch.arange(11)
    table = torch.as_tensor(cache.bm.block_table(0)[0], dtype=torch.int64)
    for pool, rows, sc in ((cache.k_cache, k, 0.5), (cache.v_cache, v, 0.25)):
        got = pool[table[t // bs].cuda(), :, (t % bs).cuda(), :].cpu().numpy()
        assert np.array_equal(got, int8.quantize(rows.float().numpy(), sc))
        assert got.min() >= -127
    assert cache.k_cache[table[0], 0, 0, :8].cpu().tolist() == [127, -127, 127, -127, 0, 0, 2, -2]
    assert cache.v_cache[table[0], 1, 3, :4].cpu().tolist() == [127, 126, -127, 0]


def test_int8_swap_round_trip_decodes_the_same():
    g = torch.Generator().manual_seed(16)
    cache = PagedKVCache(10, 4, 16, 128, torch.int8, "cuda", list(range(10)), fill=float("nan"),
                         k_scale=K_SCALE, v_scale=V_SCALE)
    cache.enable_swap(8)
    k, v = torch.randn(50, 4, 128, generator=g).bfloat16(), torch.randn(50, 4, 128, generator=g).bfloat16()
    cache.add_sequence(1, k.cuda(), v.cuda())
    q = torch.randn(1, 4, 128, generator=g).bfloat16().cuda()
    before = cache.decode([1], q, 128 ** -0.5).cpu()
    codes_before = cache.k_cache[cache.bm.block_table(1)[0].tolist()].cpu()
    cache.swap_out(1)
    junk = torch.randn(160, 4, 128, generator=g).bfloat16().cuda()
    cache.add_sequence(2, junk, junk)
    cache.free(2)
    cache.swap_in(1)
    after = cache.decode([1], q, 128 ** -0.5).cpu()
    assert torch.equal(codes_before, cache.k_cache[cache.bm.block_table(1)[0].tolist()].cpu())
    assert torch.equal(before, after)
    assert B.pa_get_device_error()[0] == B.PA_OK


def test_int8_step_host_matches_oracle():
    sh = W.Shape(16, 4, 128, 16, "bf16")
    g = torch.Generator().manual_seed(23)
    ref = OracleRun(sh, 64, list(range(64)), keep_pool=False)
    cache = PagedKVCache(64, 4, 16, 128, torch.int8, "cuda", list(range(64)), fill=float("nan"),
                         k_scale=K_SCALE, v_scale=V_SCALE)
    pk, pv = torch.randn(29, 4, 128, generator=g).bfloat16(), torch.randn(29, 4, 128, generator=g).bfloat16()
    ref.apply(("add", 0, 29, lambda which, device="cpu": pk if which == "k" else pv))
    cache.add_sequence(0, pk.cuda(), pv.cuda())
    ref.apply(("fork", 0, 1))
    cache.fork(0, 1)
    ids = [1, 0]
    for step in range(2):
        q = torch.randn(2, 16, 128, generator=g).bfloat16().pin_memory()
        k = torch.randn(2, 4, 128, generator=g).bfloat16().pin_memory()
        v = torch.randn(2, 4, 128, generator=g).bfloat16().pin_memory()
        out = torch.empty(2, 16, 128, dtype=torch.float32).pin_memory()
        ref.apply(("append", ids, lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
        cache.step_host(ids, q, k, v, out, 128 ** -0.5)
        for i, s in enumerate(ids):
            K, V = _dq(ref.history(s, "k"), K_SCALE), _dq(ref.history(s, "v"), V_SCALE)
            exp = np.concatenate([decode_attention(q[i][4 * h:4 * h + 4], K[:, h:h + 1], V[:, h:h + 1], 128 ** -0.5)
                                  for h in range(4)])
            assert float(np.abs(out[i].double().numpy() - exp).max()) <= TOL8
    assert B.pa_get_device_error()[0] == B.PA_OK


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_int8_prefill_chunked_matches_oracle(G, D, bs):
    """Chunked prefill over an int8 cache against the fp64 attention over the
    dequantised rows."""
    from oracle.prefill import prefill_attention
    rng = np.random.default_rng(9000 + G * 1000 + D + bs)
    hkv, nseq = 2, 5
    pre = rng.integers(0, 300, size=nseq)
    pre[0] = 0
    chunk = rng.integers(1, 200, size=nseq)
    chunk[1] = 128 // G
    chunk[2] = 64 // G
    chunk[3] = 256 // G + 3
    nb = int(sum(-(-int(p + c) // bs) for p, c in zip(pre, chunk))) + 4
    cache = PagedKVCache(nb, hkv, bs, D, torch.int8, "cuda", rng.permutation(nb), fill=float("nan"),
                         k_scale=K_SCALE, v_scale=V_SCALE)
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
        ref = prefill_attention(q[row:row + n], _dq(K[s], K_SCALE), _dq(V[s], V_SCALE), D ** -0.5)
        o = out[row:row + n].double().numpy()
        assert np.isfinite(o).all()
        err = float(np.abs(o - ref).max())
        assert err <= TOL8, f"seq {s}: {err}"
        row += n

