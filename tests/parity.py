"""Shared driver for the GPU parity tests: replays one operation script on the
CUDA path (PagedKVCache -> libpagedattn) and on the oracle, and compares.

Tolerances (max-abs against the fp64 oracle): fp32 caches 1e-5, bf16 caches
4e-3; both accumulate in fp32 on the GPU. Slots, copy-on-write pairs, block
tables and cached bytes must match exactly.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle.attention import decode_attention
from oracle.replay import OracleRun
from paged_kv_cache_361_b200 import PagedKVCache, binding as B
from paged_kv_cache_361_b200 import workloads as W

TOL = {"f32": 1e-5, "bf16": 4e-3}


def bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def oracle_rows(run: OracleRun, seq: int, q_row: torch.Tensor, scale: float, use_pool=False) -> np.ndarray:
    """fp64 output [Hq][D], one kv group at a time (keeps fp64 copies small)."""
    sh = run.shape
    K, V = (run.paged_rows(seq, w) for w in "kv") if use_pool else (run.history(seq, w) for w in "kv")
    G = sh.group
    out = np.zeros((sh.num_q_heads, sh.head_dim))
    for g in range(sh.num_kv_heads):
        out[g * G:(g + 1) * G] = decode_attention(q_row[g * G:(g + 1) * G], K[:, g:g + 1], V[:, g:g + 1], scale)
    return out


class Replay:
    """Runs the script on both sides, op by op."""

    def __init__(self, shape: W.Shape, num_blocks: int, free_order, scale: float, device="cuda",
                 partition_tokens: int = -1, keep_pool: bool = True, fill=float("nan")):
        self.shape, self.scale, self.P = shape, scale, partition_tokens
        self.cache = PagedKVCache(num_blocks, shape.num_kv_heads, shape.block_size, shape.head_dim,
                                  W.TORCH_DTYPE[shape.dtype], device, free_order, fill=fill)
        self.oracle = OracleRun(shape, num_blocks, free_order, keep_pool=keep_pool, pool_fill=fill)
        self.device = device
        self.decodes = []      # (ids, q_cpu, out_gpu_cpu)
        self.n_pairs = 0

    def apply(self, op, check_decode=None):
        kind = op[0]
        rec = self.oracle.apply(op)
        if kind == "add":
            _, seq, n, src = op
            slots = self.cache.add_sequence(seq, src("k").to(self.device), src("v").to(self.device))
            assert slots.tolist() == rec["slots"]
        elif kind == "add_cached":
            _, seq, tokens, src = op
            slots, n_cached = self.cache.add_sequence_cached(seq, tokens, src("k").to(self.device),
                                                             src("v").to(self.device))
            assert slots.tolist() == rec["slots"] and n_cached == rec["n_cached"]
            self.n_cached = getattr(self, "n_cached", 0) + n_cached
        elif kind == "fork":
            self.cache.fork(op[1], op[2])
        elif kind == "append":
            _, ids, src = op
            slots, pairs = self.cache.append(ids, src("k").to(self.device), src("v").to(self.device))
            assert slots.tolist() == rec["slots"]
            assert pairs.tolist() == [list(p) for p in rec["pairs"]]
            self.n_pairs += len(pairs)
        elif kind == "free":
            self.cache.free(op[1])
        elif kind == "decode":
            _, ids, qsrc = op
            q = qsrc()
            tables, lens, _ = self.cache.decode_inputs(ids)
            for i, s in enumerate(ids):
                assert tables[i, :len(rec["tables"][i])].tolist() == rec["tables"][i]
                assert lens[i] == rec["lens"][i]
            out = self.cache.decode(ids, q.to(self.device), self.scale, partition_tokens=self.P)
            self.decodes.append((list(ids), q, out.cpu()))
        return rec

    def run(self, ops):
        for op in ops:
            self.apply(op)
        torch.cuda.synchronize()
        st, info = B.pa_get_device_error()
        assert st == B.PA_OK, (st, info)
        return self

    def check_outputs(self, which=-1, seqs=None, tol=None):
        """Max-abs error of decode `which` against the oracle history."""
        ids, q, out = self.decodes[which]
        tol = TOL[self.shape.dtype] if tol is None else tol
        worst = 0.0
        for i, s in enumerate(ids):
            if seqs is not None and i not in seqs:
                continue
            ref = oracle_rows(self.oracle, s, q[i], self.scale)
            err = float(np.abs(out[i].double().numpy() - ref).max())
            assert np.isfinite(out[i].numpy()).all(), f"non-finite output for seq {s}"
            worst = max(worst, err)
            assert err <= tol, f"seq {s}: max-abs {err:.3e} > {tol}"
        return worst

    def check_pool_rows(self, seqs=None):
        """Every live sequence's rows, read from the device pool through the C++
        table, equal its contiguous history bitwise."""
        kc, vc = self.cache.k_cache, self.cache.v_cache
        bs = self.shape.block_size
        for s in (self.cache.lens if seqs is None else seqs):
            table, L = self.cache.bm.block_table(s)
            t = torch.arange(L)
            blk = torch.as_tensor(table, dtype=torch.int64)[t // bs].to(kc.device)
            off = (t % bs).to(kc.device)
            for w, pool in (("k", kc), ("v", vc)):
                got = pool[blk, :, off, :].cpu()
                ref = self.oracle.history(s, w)
                assert torch.equal(bits(got), bits(ref)), f"seq {s} {w} rows differ"

    def check_pool_bitwise(self):
        """Whole device pool equals the oracle's paged pool (small cases)."""
        for w, pool in (("k", self.cache.k_cache), ("v", self.cache.v_cache)):
            assert torch.equal(bits(pool.cpu()), bits(self.oracle.pool[w]))


# 8-bit caches: torch dtype, oracle codec module, integer view of the pool bytes
def _codecs():
    from oracle import fp8, int8
    return {"e4m3": (torch.float8_e4m3fn, fp8, torch.uint8), "int8": (torch.int8, int8, torch.int8)}


class CodedReplay(Replay):
    """Replay with an 8-bit device cache (e4m3 or int8 codes, per-tensor
    scales); the oracle keeps the bf16 history and quantises it itself."""

    def __init__(self, shape, num_blocks, free_order, scale, partition_tokens=-1, k_scale=4.0 / 448.0,
                 v_scale=3.0 / 448.0, fmt="e4m3"):
        assert shape.dtype == "bf16"
        self.shape, self.scale, self.P = shape, scale, partition_tokens
        self.ks, self.vs = k_scale, v_scale
        self.dt, self.codec, self.view = _codecs()[fmt]
        self.cache = PagedKVCache(num_blocks, shape.num_kv_heads, shape.block_size, shape.head_dim,
                                  self.dt, "cuda", free_order, fill=float("nan"),
                                  k_scale=k_scale, v_scale=v_scale)
        self.oracle = OracleRun(shape, num_blocks, free_order, keep_pool=False)
        self.device = "cuda"
        self.decodes = []
        self.n_pairs = 0

    def codes(self, seq, which):
        return self.codec.quantize(self.oracle.history(seq, which).float().numpy(),
                                   self.ks if which == "k" else self.vs)

    def rows(self, seq, which):
        return self.codec.dequantize(self.codes(seq, which), self.ks if which == "k" else self.vs)

    def check_pool_codes(self):
        bs = self.shape.block_size
        for s in self.cache.lens:
            table, L = self.cache.bm.block_table(s)
            t = torch.arange(L)
            blk = torch.as_tensor(table, dtype=torch.int64)[t // bs].cuda()
            off = (t % bs).cuda()
            for w, pool in (("k", self.cache.k_cache), ("v", self.cache.v_cache)):
                got = pool.view(self.view)[blk, :, off, :].cpu().numpy()
                assert np.array_equal(got, self.codes(s, w)), f"seq {s} {w} codes differ"

    def check_outputs(self, which=-1, tol=TOL["bf16"]):
        """Outputs are fp32 sums over exactly representable inputs (codes times
        a scale, bf16 queries), as for a bf16 cache: the bf16 bound applies."""
        ids, q, out = self.decodes[which]
        G = self.shape.group
        worst = 0.0
        for i, s in enumerate(ids):
            K, V = self.rows(s, "k"), self.rows(s, "v")
            ref = np.zeros((self.shape.num_q_heads, self.shape.head_dim))
            for g in range(self.shape.num_kv_heads):
                ref[g * G:(g + 1) * G] = decode_attention(q[i][g * G:(g + 1) * G], K[:, g:g + 1], V[:, g:g + 1],
                                                          self.scale)
            o = out[i].double().numpy()
            assert np.isfinite(o).all()
            err = float(np.abs(o - ref).max())
            worst = max(worst, err)
            assert err <= tol, f"seq {s}: max-abs {err:.3e} > {tol}"
        return worst
