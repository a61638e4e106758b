"""GPU parity of the e4m3 KV cache (per-tensor K and V scales, bf16 inputs)
against the oracle: the codes pa_reshape_and_cache stores are compared bit for
bit with oracle/fp8.py's quantiser, and pa_decode with the fp64 attention over
the oracle's dequantised rows. Block copies and swaps move codes unchanged."""
import zlib

import numpy as np
import pytest
import torch

from oracle import fp8
from oracle.attention import decode_attention
from oracle.replay import OracleRun
from paged_kv_cache_361_b200 import PagedKVCache, binding as B
from paged_kv_cache_361_b200 import workloads as W
from tests.parity import CodedReplay

pytestmark = pytest.mark.gpu

# Outputs are fp32 sums over exactly representable inputs (e4m3 codes times a
# scale, bf16 queries), as for a bf16 cache: the bf16 bound applies.
TOL_FP8 = 4e-3
# N(0, 1) rows: |x| up to 4 uses the whole e4m3 range; rarer larger values saturate
K_SCALE, V_SCALE = 4.0 / 448.0, 3.0 / 448.0


@pytest.fixture(autouse=True)
def _clean_error_word():
    if torch.cuda.is_available():
        B.pa_get_device_error()
    yield


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_fp8_fuzz_shapes(D, G, bs):
    hkv = 2
    sh = W.Shape(hkv * G, hkv, D, bs, "bf16")
    seed = zlib.crc32(f"fp8-{D}-{G}-{bs}".encode()) % 100000
    w = W.random_small(seed, num_seqs=6, shape=sh, max_len=int(np.random.default_rng(seed).integers(40, 400)))
    for P in (0, -1, 2 * max(bs, 16)):
        r = CodedReplay(sh, w.num_blocks, w.free_order, w.scale, partition_tokens=P).run(W.simple_ops(w))
        r.check_outputs()
    r.check_pool_codes()


def test_fp8_long_split_and_mha():
    """Llama-2-7B-shaped heads (32 x 128, MHA) and a 4k-token sequence cut into
    partitions, against the oracle."""
    sh = W.Shape(32, 32, 128, 16, "bf16")
    w = W.random_small(21, num_seqs=3, shape=sh, max_len=4096)
    for P in (0, 512, -1):
        r = CodedReplay(sh, w.num_blocks, w.free_order, w.scale, partition_tokens=P).run(W.simple_ops(w))
        r.check_outputs()
    r.check_pool_codes()


def test_fp8_fork_copy_on_write():
    """Samples forked from one prompt share its blocks; the first append copies
    the shared partial block (a byte copy of codes) before writing."""
    sh = W.Shape(8, 2, 128, 16, "bf16")
    g = torch.Generator().manual_seed(8)
    pk, pv = torch.randn(37, 2, 128, generator=g).bfloat16(), torch.randn(37, 2, 128, generator=g).bfloat16()
    ops = [("add", 0, 37, lambda which, device="cpu": pk if which == "k" else pv),
           ("fork", 0, 1), ("fork", 0, 2)]
    for step in range(5):
        k, v = torch.randn(3, 2, 128, generator=g).bfloat16(), torch.randn(3, 2, 128, generator=g).bfloat16()
        ops.append(("append", [2, 0, 1], lambda which, device="cpu", k=k, v=v: k if which == "k" else v))
    q = torch.randn(3, 8, 128, generator=g).bfloat16()
    ops.append(("decode", [0, 1, 2], lambda device="cpu": q))
    r = CodedReplay(sh, 20, list(range(20)), 128 ** -0.5).run(ops)
    assert r.n_pairs == 2
    r.check_pool_codes()
    r.check_outputs()


def test_fp8_reshape_saturates_and_keeps_nan():
    """Values past the e4m3 range saturate to +-448 * scale; NaN stays NaN; the
    codes equal the oracle's bit for bit (a NaN code only as a NaN code)."""
    hkv, D, bs = 2, 64, 8
    cache = PagedKVCache(4, hkv, bs, D, torch.float8_e4m3fn, "cuda", list(range(4)), fill=0.0,
                         k_scale=0.5, v_scale=0.01)
    g = torch.Generator().manual_seed(4)
    k = (torch.randn(11, hkv, D, generator=g) * 100).bfloat16()
    v = torch.randn(11, hkv, D, generator=g).bfloat16()
    k[0, 0, :6] = torch.tensor([float("inf"), -float("inf"), 1e30, -1e30, float("nan"), 224.0 * 0.5 * 1.03])
    v[3, 1, :3] = torch.tensor([4.48, 4.49, -100.0])
    cache.add_sequence(0, k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert B.pa_get_device_error()[0] == B.PA_OK
    t = torch.arange(11)
    table = torch.as_tensor(cache.bm.block_table(0)[0], dtype=torch.int64)
    for pool, rows, sc in ((cache.k_cache, k, 0.5), (cache.v_cache, v, 0.01)):
        got = pool.view(torch.uint8)[table[t // bs].cuda(), :, (t % bs).cuda(), :].cpu().numpy()
        exp = fp8.quantize(rows.float().numpy(), sc)
        nan = (exp & 0x7F) == 0x7F
        assert np.array_equal(got[~nan], exp[~nan])
        assert np.all((got[nan] & 0x7F) == 0x7F)
    assert (got == 0xFF).sum() + (got == 0x7F).sum() == 0   # the v rows carry no NaN


def test_fp8_swap_round_trip_decodes_the_same():
    g = torch.Generator().manual_seed(6)
    sh = W.Shape(4, 4, 128, 16, "bf16")
    cache = PagedKVCache(10, 4, 16, 128, torch.float8_e4m3fn, "cuda", list(range(10)), fill=float("nan"),
                         k_scale=K_SCALE, v_scale=V_SCALE)
    cache.enable_swap(8)
    k, v = torch.randn(50, 4, 128, generator=g).bfloat16(), torch.randn(50, 4, 128, generator=g).bfloat16()
    cache.add_sequence(1, k.cuda(), v.cuda())
    q = torch.randn(1, 4, 128, generator=g).bfloat16().cuda()
    before = cache.decode([1], q, 128 ** -0.5).cpu()
    codes_before = cache.k_cache.view(torch.uint8)[cache.bm.block_table(1)[0].tolist()].cpu()
    cache.swap_out(1)
    junk = torch.randn(160, 4, 128, generator=g).bfloat16().cuda()
    cache.add_sequence(2, junk, junk)
    cache.free(2)
    cache.swap_in(1)
    after = cache.decode([1], q, 128 ** -0.5).cpu()
    assert torch.equal(codes_before, cache.k_cache.view(torch.uint8)[cache.bm.block_table(1)[0].tolist()].cpu())
    assert torch.equal(before, after)
    assert B.pa_get_device_error()[0] == B.PA_OK


def test_fp8_step_host_matches_oracle():
    sh = W.Shape(16, 4, 128, 16, "bf16")
    g = torch.Generator().manual_seed(13)
    ref = OracleRun(sh, 64, list(range(64)), keep_pool=False)
    cache = PagedKVCache(64, 4, 16, 128, torch.float8_e4m3fn, "cuda", list(range(64)), fill=float("nan"),
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
            K = fp8.dequantize(fp8.quantize(ref.history(s, "k").float().numpy(), K_SCALE), K_SCALE)
            V = fp8.dequantize(fp8.quantize(ref.history(s, "v").float().numpy(), V_SCALE), V_SCALE)
            exp = np.concatenate([decode_attention(q[i][4 * h:4 * h + 4], K[:, h:h + 1], V[:, h:h + 1], 128 ** -0.5)
                                  for h in range(4)])
            assert float(np.abs(out[i].double().numpy() - exp).max()) <= TOL_FP8
    assert B.pa_get_device_error()[0] == B.PA_OK


def _dq(x, scale):
    """The oracle's view of bf16 rows stored in an e4m3 cache: dequantised codes (fp64)."""
    return fp8.dequantize(fp8.quantize(x.float().numpy(), scale), scale)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fp8_prefill_chunked_matches_oracle(G, D, bs):
    """Chunked prefill over an e4m3 cache: sequences grow by a chunk or start;
    every new token's causal attention matches the oracle's fp64 attention over
    the dequantised rows. Pool padding is NaN codes."""
    from oracle.prefill import prefill_attention
    rng = np.random.default_rng(7000 + G * 1000 + D + bs)
    hkv, nseq = 2, 5
    pre = rng.integers(0, 300, size=nseq)
    pre[0] = 0
    chunk = rng.integers(1, 200, size=nseq)
    chunk[1] = 128 // G           # exactly one 128-row query tile
    chunk[2] = 64 // G            # half a tile
    chunk[3] = 256 // G + 3       # two tiles (one CTA at head_dim 128) and a ragged third
    nb = int(sum(-(-int(p + c) // bs) for p, c in zip(pre, chunk))) + 4
    cache = PagedKVCache(nb, hkv, bs, D, torch.float8_e4m3fn, "cuda", rng.permutation(nb), fill=float("nan"),
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
        assert err <= TOL_FP8, f"seq {s}: {err}"
        row += n


@pytest.mark.parametrize("G,D", [(1, 128), (8, 128), (4, 64)])
def test_fp8_prefill_long_chunk_many_tiles(G, D):
    """A 700-token chunk after 900 cached tokens over an e4m3 cache: many query
    tiles, 25 key chunks, a ragged last tile and key chunk (sampled rows)."""
    from oracle.prefill import prefill_attention
    hkv, bs = 2, 16
    g = torch.Generator().manual_seed(90 + G + D)
    pre, n = 900, 700
    nb = -(-(pre + n) // bs) + 3
    cache = PagedKVCache(nb, hkv, bs, D, torch.float8_e4m3fn, "cuda", np.random.default_rng(G).permutation(nb),
                         fill=float("nan"), k_scale=K_SCALE, v_scale=V_SCALE)
    K = torch.randn(pre + n, hkv, D, generator=g).bfloat16()
    V = torch.randn(pre + n, hkv, D, generator=g).bfloat16()
    cache.add_sequence(0, K[:pre].cuda(), V[:pre].cuda())
    q = torch.randn(n, hkv * G, D, generator=g).bfloat16()
    out = cache.prefill([0], [n], q.cuda(), K[pre:].cuda(), V[pre:].cuda(), D ** -0.5).cpu()
    assert B.pa_get_device_error()[0] == B.PA_OK
    rows = np.r_[0:30, 300:330, n - 30:n]
    ref = prefill_attention(q, _dq(K, K_SCALE), _dq(V, V_SCALE), D ** -0.5)
    err = float(np.abs(out.double().numpy()[rows] - ref[rows]).max())
    assert err <= TOL_FP8, err


def test_fp8_bad_scale_rejected():
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.float8_e4m3fn, device="cuda")
    vc = torch.zeros_like(kc)
    B.set_kv_scales(kc, vc, 0.0, 1.0)
    rows = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device="cuda")
    slots = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(B.PagedAttnError) as e:
        B.pa_reshape_and_cache(rows, rows, slots, kc, vc)
    assert e.value.status == B.PA_ERR_INVALID_ARG
