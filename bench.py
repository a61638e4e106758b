#!/usr/bin/env python
"""Decode-step benchmark of libpagedattn on the Llama-2-7B-shaped workload.

Workload: 64 sequences, context lengths uniform in [128, 2048] before the step
(one token appended, then decode), 32 query heads = 32 kv heads, head_dim 128,
block_size 16, bf16 cache, pool = 1.1 x blocks needed with ids in a seeded
shuffle, Q/K/V ~ N(0, 1). One step = the whole hot path for one batch: the
KV append and decode attention in one launch (pa_decode_append: the decode
CTAs write the step's new K/V rows at their slots), split into partitions with
its log-sum-exp merge when the library chooses to.

Metric: KV bytes read by decode per second (GB/s, fraction of HBM peak), and
decode tokens per second. The 1.07 GB of K/V read per step is far larger than
the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (the path has no exchange
step), one per GPU; value = all ranks' bytes / max over ranks of the time.
`--impl reference` times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-decode KV-read GB/s (% of B200 HBM peak); decode attention tokens/sec"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one call of the
# timed operation (every kernel of pa_decode / pa_decode_cascade / pa_prefill),
# from one-pass ncu launch lists of this script (averaged over the listed
# launches), keyed by (workload, cache dtype, partition tokens, path). Each
# entry names the library sources of those kernels and their hash at capture:
# an entry whose files have changed since is stale and reported as null, as is
# any configuration without a capture. The command lines are in profiles/.
_DEC = ["common.cuh", "decode_common.cuh", "capi.cu"]
_PF = ["common.cuh", "decode_common.cuh", "decode_f8.cuh", "prefill_mma.cuh", "prefill_tc.cuh", "tcgen05.cuh",
       "capi.cu"]
NCU_TRAFFIC: dict = {
    ("llama2_7b_mha", "bfloat16", 0, "decode"): dict(
        bytes=1_079_387_221 + 2_192_299, files=_DEC + ["decode_simt.cuh"], sha="8e318919c2abc840",
        note="decode_simt_kernel of pa_decode_append (the step's only launch), 3 launches"),
    ("llama2_7b_mha", "float8_e4m3fn", 0, "decode"): dict(
        bytes=540_502_443 + 1_836_459, files=_DEC + ["decode_f8.cuh"], sha="5ff75b7b610d5d43",
        note="decode_f8_kernel (e4m3) of pa_decode_append, 3 launches"),
    ("llama2_7b_mha", "int8", 0, "decode"): dict(
        bytes=540_523_947 + 1_852_928, files=_DEC + ["decode_f8.cuh"], sha="5ff75b7b610d5d43",
        note="decode_f8_kernel (int8) of pa_decode_append, 3 launches"),
    ("long_context_split", "bfloat16", 512, "decode"): dict(
        bytes=1_343_030_613 + 6_136_832 + 21_471_744, files=_DEC + ["decode_mma.cuh"], sha="572fd0d77d91b599",
        note="decode_mma_persistent_kernel + decode_reduce_kernel, 3 launches each"),
    ("parallel_sampling", "bfloat16", 0, "decode"): dict(
        bytes=113_622_400 + 601_728, files=_DEC + ["decode_mma.cuh"], sha="572fd0d77d91b599",
        note="decode_mma_kernel of pa_decode_append, 6 launches (1.17x the 97.5 MB of distinct blocks: with the "
             "longest-first order a prompt's samples no longer all run at once)"),
    ("parallel_sampling", "bfloat16", 0, "cascade"): dict(
        bytes=32_022_272 + 768 + 72_888_013 + 103_168, files=_DEC + ["decode_mma.cuh", "prefill_mma.cuh"], sha="de27b89ffdac9c43",
        note="prefill_mma_kernel (prefix pass) + decode_mma_kernel (suffixes and fold), 5-6 launches each"),
    ("continuous_batching", "bfloat16", 0, "decode"): dict(
        bytes=835_087_625 + 2_439_945, files=_DEC + ["decode_mma.cuh"], sha="572fd0d77d91b599",
        note="decode_mma_kernel of pa_decode_append over steps 0-29 of the trace (32768-block pool); their "
             "algorithmic mean is 825.0 MB per step (x1.015), the 200-step mean 811.2 MB"),
    ("prefill_llama2_7b_mha", "bfloat16", 0, "prefill"): dict(
        bytes=1_308_881_000 + 228_545_280, files=_PF, sha="de28dba00f317626",
        how="ncu capture (the profile's metric set, one launch)", note="prefill_tc_kernel, 1 launch (Q, K/V per tile pair not served by L2, the fp32 output)"),
    ("prefill_llama2_7b_mha", "float8_e4m3fn", 0, "prefill"): dict(
        bytes=662_598_656 + 226_810_368, files=_PF, sha="de28dba00f317626", how="ncu capture (the profile's metric set, one launch)", note="prefill_tc_kernel (e4m3), 1 launch"),
    ("prefill_gqa8", "bfloat16", 0, "prefill"): dict(
        bytes=758_603_264 + 483_280_640, files=_PF, sha="de28dba00f317626", how="ncu capture (the profile's metric set, one launch)", note="prefill_tc_kernel, 1 launch"),
}
CSRC = os.path.join(ROOT, "paged_kv_cache_361_b200", "csrc")


def src_hash(files) -> str:
    """sha256 (16 hex digits) over the named CUDA sources of the library."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(key):
    e = NCU_TRAFFIC.get(key)
    if e is None:
        return None, "no capture of this configuration"
    if src_hash(e["files"]) != e["sha"]:
        return None, "stale: the kernels' sources changed since the capture"
    how = e.get("how", "one-pass ncu launch list")
    return e["bytes"], f"{how} of the current kernels (sources {e['sha']}): {e['note']}"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# --- ranks -------------------------------------------------------------------------

def combine_ranks(ms: float, nbytes: float, world: int, device) -> tuple[float, float]:
    """Whole-job figures of a replicated run: the slowest rank's time and the
    bytes of all ranks (one float64 all-reduce each; no-op for one rank)."""
    if world <= 1:
        return float(ms), float(nbytes)
    tm = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    tb = torch.tensor([float(nbytes)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(tm, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(tb, op=torch.distributed.ReduceOp.SUM)
    return float(tm.item()), float(tb.item())


# --- clocks sampling -------------------------------------------------------------

class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        except Exception:
            bus = None
        self.sel = bus

    def start(self):
        try:
            import tempfile
            self.path = os.path.join(tempfile.gettempdir(), f"pa_bench_clocks_{os.getpid()}.csv")
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if self.sel:
                cmd += ["-i", self.sel]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --- workload --------------------------------------------------------------------

WORKLOADS = {
    "llama2_7b_mha": "llama2_7b_mha_decode: 64 seqs, ctx U[128,2048]+1, 32/32 heads, D128, bs16, bf16",
    "long_context_split": "long_context_split_decode: 4 seqs, ctx 32768/65536/98304/131072+1, 64/8 heads, D128, bs32, "
                          "512-token partitions, bf16",
    "parallel_sampling": "parallel_sampling_decode: 8 prompts x 8 samples, 1000-token shared prefix + tails U[1,512], "
                         "32/8 heads, D128, bs16, bf16",
    "continuous_batching": "continuous_batching_decode: 256 live seqs, ctx lognormal(500,1) capped 4096, all 200 steps "
                           "of the trace (finish p 0.005, arrivals lognormal(300,1)), 200k-block pool, 32/8 heads, D128, "
                           "bs16, bf16",
}


def workload_ops(name, seed):
    """(shape, num_blocks, free_order, scale, partition_tokens, ops) of a workload;
    the last two ops are the measured step's append and decode."""
    from paged_kv_cache_361_b200 import workloads as W
    if name in ("llama2_7b_mha", "long_context_split"):
        w = W.llama2_7b_mha(seed=seed) if name == "llama2_7b_mha" else W.long_context_split(seed=seed)
        return w.shape, w.num_blocks, w.free_order, w.scale, w.partition_tokens, W.simple_ops(w)
    if name == "parallel_sampling":
        w = W.parallel_sampling(seed=seed)
        return w.shape, w.num_blocks, w.free_order, w.scale, 0, W.sampling_ops(w, batch_tail_steps=True)
    tr = W.continuous_batching(seed=seed)
    return tr.shape, tr.num_blocks, tr.free_order, 1.0 / math.sqrt(tr.shape.head_dim), 0, W.batching_ops(tr, steps=1)


def fill_pool(cache, nb, kv_dtype, g, device):
    """Device-generated pool contents standing in for the prompts' K/V: N(0,1)
    values (bf16, or e4m3 codes at scale 1), or uniform int8 codes."""
    for t in (cache.k_cache, cache.v_cache):
        for i in range(0, nb, 1024):   # chunked to bound the fp32 temporary
            if kv_dtype == "int8":
                t[i:i + 1024] = torch.randint(-127, 128, t[i:i + 1024].shape, generator=g, device=device,
                                              dtype=torch.int8)
            else:
                t[i:i + 1024] = torch.randn(t[i:i + 1024].shape, generator=g, device=device).to(t.dtype)


def make_cache(sh, nb, order, kv_dtype, device):
    from paged_kv_cache_361_b200 import PagedKVCache
    from paged_kv_cache_361_b200 import workloads as W
    dt = W.TORCH_DTYPE[sh.dtype]
    cache_dt = {"fp8": torch.float8_e4m3fn, "int8": torch.int8}.get(kv_dtype, dt)
    sc = 4.0 / 127 if kv_dtype == "int8" else 1.0
    return PagedKVCache(nb, sh.num_kv_heads, sh.block_size, sh.head_dim, cache_dt, device, order, k_scale=sc,
                        v_scale=sc), dt


def build_workload(seed: int, device, name: str = "llama2_7b_mha", kv_dtype: str = "auto"):
    """Replays the workload's operation script up to the measured step through
    PagedKVCache: the pool is filled with N(0,1) values on the device (they
    stand in for the prompts' K/V, so prefills only reserve blocks), forks
    share blocks, earlier appends write random rows (with their copy-on-write
    block copies). The measured step's slots and pairs come from the C++ block
    manager; its tables and lengths are uploaded once.

    kv_dtype "fp8" stores the cache as e4m3 codes (per-tensor scales 1.0: the
    N(0,1) values are inside the e4m3 range), "int8" as uniform random int8
    codes in [-127, 127] (scales 4/127); q and the new K/V rows stay bf16."""
    sh, nb, order, scale, part, ops = workload_ops(name, seed)
    cache, dt = make_cache(sh, nb, order, kv_dtype, device)
    g = torch.Generator(device=device)
    g.manual_seed(1000 + seed)
    fill_pool(cache, nb, kv_dtype, g, device)
    hkv, D = sh.num_kv_heads, sh.head_dim
    assert ops[-2][0] == "append" and ops[-1][0] == "decode"
    for op in ops[:-2]:
        if op[0] == "add":
            cache.reserve(op[1], op[2])
        elif op[0] == "fork":
            cache.fork(op[1], op[2])
        elif op[0] == "free":
            cache.free(op[1])
        elif op[0] == "append":
            n = len(op[1])
            cache.append(op[1], torch.randn((n, hkv, D), generator=g, device=device).to(dt),
                         torch.randn((n, hkv, D), generator=g, device=device).to(dt))
    ids = list(ops[-1][1])
    slots, pairs = cache.bm.append_slots(ids)
    for s in ids:
        cache.lens[s] += 1
    tables, lens32, max_len = cache.decode_inputs(ids)
    B_, hq = len(ids), sh.num_q_heads
    eb = cache.k_cache.element_size()
    st = cache.bm.stats()
    return dict(
        name=name, shape=sh, scale=scale, part=part, ids=ids, cache=cache, bm=cache.bm, kc=cache.k_cache,
        vc=cache.v_cache,
        q=torch.randn((B_, hq, D), generator=g, device=device).to(dt),
        k=torch.randn((B_, hkv, D), generator=g, device=device).to(dt),
        v=torch.randn((B_, hkv, D), generator=g, device=device).to(dt),
        slots=torch.from_numpy(slots).to(device),
        pairs=torch.from_numpy(pairs).to(device) if len(pairs) else None,
        # dispatch order of the decode CTAs: longest sequence first (C++ block manager)
        order=torch.from_numpy(cache.bm.longest_first(ids)).to(device),
        tables=torch.from_numpy(tables).to(device),
        lens=torch.from_numpy(lens32).to(device),
        lens_host=lens32.astype(np.int64),
        out=torch.empty((B_, hq, D), dtype=torch.float32, device=device),
        max_len=max_len,
        kv_bytes=int(lens32.astype(np.int64).sum()) * hkv * D * 2 * eb,
        unique_kv_bytes=int(st["used_slots"]) * hkv * D * 2 * eb,
    )


def cascade_inputs(d, device):
    """Group arguments of pa_decode_cascade for the measured step (host work
    done once, before timing), from the C++ block manager
    (pa_bm_prefix_groups): sequences whose tables start with the same blocks
    share their common prefix; the suffix CTAs go longest first
    (pa_bm_longest_first)."""
    from paged_kv_cache_361_b200 import binding as B
    cache, sh = d["cache"], d["shape"]
    offs, members, prefix, seq_prefix, max_pre = cache.shared_prefix_groups(d["ids"], 64 // sh.group)
    order = cache.bm.longest_first(d["ids"], seq_prefix)
    nbytes = B.pa_decode_cascade_workspace_bytes(len(d["ids"]), sh.num_q_heads, sh.num_kv_heads, sh.head_dim,
                                                 d["max_len"], sh.block_size, max_pre)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    # (..., workspace, stream, seq_order) of binding.pa_decode_cascade
    return (t(offs), t(members), t(prefix), t(seq_prefix), int(max(np.diff(offs), default=0)), max_pre, ws, None,
            t(order))


def sample_rows(d, seqs):
    """Host copies (before any kernel runs) of the sampled sequences' K/V rows,
    read from the device pool through their block tables: input to the CPU
    baseline only."""
    bm = d["bm"]
    bs = d["shape"].block_size
    rows = []
    for s in seqs:
        table, L = bm.block_table(d["ids"][s])
        L_old = L - 1
        t = torch.arange(L_old)
        blk = torch.as_tensor(table, dtype=torch.int64)[t // bs].to(d["kc"].device)
        off = (t % bs).to(d["kc"].device)
        K = torch.cat([d["kc"][blk, :, off, :].float(), d["k"][s:s + 1].float()]).cpu()
        V = torch.cat([d["vc"][blk, :, off, :].float(), d["v"][s:s + 1].float()]).cpu()
        rows.append((s, K, V, d["q"][s].cpu()))
    return rows


def time_oracle(rows, scale, budget_s, elem_bytes=2):
    """Runs the CPU oracle over the sampled sequences (repeating the sample)
    until budget_s has passed; returns (GB/s, seconds, sequences done); bytes
    are counted at the cache's element size."""
    from oracle.attention import decode_attention
    done_bytes, n, t0 = 0, 0, time.perf_counter()
    while True:
        for s, K, V, q in rows:
            decode_attention(q, K, V, scale)
            done_bytes += K.numel() * elem_bytes * 2
            n += 1
            if time.perf_counter() - t0 >= budget_s:
                el = time.perf_counter() - t0
                return done_bytes / el / 1e9, el, n


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if blas:
            return int(max(blas))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline_record(rows, scale, seconds, elem_bytes, sample_desc):
    """The oracle on all of the BLAS pool's threads and on one thread (the
    pool limited by threadpoolctl), each for about `seconds`."""
    import threadpoolctl
    cores = cpu_threads()
    gbs, el, n = time_oracle(rows, scale, seconds, elem_bytes)
    with threadpoolctl.threadpool_limits(limits=1, user_api="blas"):
        gbs1, el1, n1 = time_oracle(rows, scale, seconds, elem_bytes)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 NumPy oracle over {sample_desc}, repeated for {el:.1f} s ({n} sequence passes) on "
                      f"{cores} BLAS threads and {el1:.1f} s ({n1} passes) on 1 thread; host has "
                      f"{os.cpu_count()} cores",
            "by_threads": {str(cores): round(gbs, 4), "1": round(gbs1, 4)}}


# --- timing helpers --------------------------------------------------------------

def ev():
    return torch.cuda.Event(enable_timing=True)


def time_calls(pre, timed, steps, warmup, stream):
    """Runs pre(); timed() `warmup` times untimed, then `steps` times with CUDA
    events around each timed() on `stream`. Returns (per-call ms list, whole
    region ms)."""
    for _ in range(warmup):
        pre()
        timed()
    torch.cuda.synchronize()
    evs = [(ev(), ev()) for _ in range(steps)]
    t0, t1 = ev(), ev()
    t0.record(stream)
    for i in range(steps):
        pre()
        evs[i][0].record(stream)
        timed()
        evs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs], t0.elapsed_time(t1)


def check_device(B, what):
    st, info = B.pa_get_device_error()
    if st != B.PA_OK:
        raise RuntimeError(f"device error {st} ({info}) in {what}")


# --- arms --------------------------------------------------------------------------

def decode_fns(B, d, P, cascade=None):
    """(pre, timed) of one decode step: the copy-on-write copies, then either
    pa_decode_append (the KV append done by the decode CTAs, one launch) or,
    for the cascade, pa_reshape_and_cache followed by pa_decode_cascade."""
    def write_step():
        if d["pairs"] is not None:
            B.pa_copy_blocks(d["kc"], d["vc"], d["pairs"])
        if cascade is not None:
            B.pa_reshape_and_cache(d["k"], d["v"], d["slots"], d["kc"], d["vc"])

    sh = d["shape"]
    nseq = len(d["ids"])
    ws_bytes = B.pa_decode_workspace_bytes(nseq, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, d["max_len"],
                                           sh.block_size, P)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=d["kc"].device)

    def decode():
        if cascade is not None:
            B.pa_decode_cascade(d["q"], d["kc"], d["vc"], d["tables"], d["lens"], d["scale"], d["out"], d["max_len"],
                                *cascade)
            return
        B.pa_decode_append(d["q"], d["k"], d["v"], d["slots"], d["kc"], d["vc"], d["tables"], d["lens"], d["scale"],
                           d["out"], d["max_len"], P, ws, seq_order=d["order"])
    return write_step, decode


def run_ours(args, rank, world, device):
    from paged_kv_cache_361_b200 import binding as B
    if args.workload == "continuous_batching":
        return run_batching_line(args, rank, world, device)
    d = build_workload(seed=rank, device=device, name=args.workload, kv_dtype=args.kv_dtype)
    sh = d["shape"]
    nseq = len(d["ids"])
    cascade = cascade_inputs(d, device) if args.cascade else None
    P = args.partition if args.partition != -2 else d["part"]
    # the cascade resolves -1 as pa_decode does; the ordered decode as pa_decode_ordered does
    P_eff = P if P >= 0 else (B.pa_decode_partition_tokens if args.cascade else B.pa_decode_ordered_partition_tokens)(
        nseq, sh.num_q_heads, sh.num_kv_heads, d["max_len"], sh.block_size)
    split = P_eff > 0 and math.ceil(d["max_len"] / P_eff) > 1
    stream = torch.cuda.current_stream(device)

    sample_seqs = [0, 1, 2, 3] if args.workload == "llama2_7b_mha" else [0]
    baseline_rows = sample_rows(d, sample_seqs) if rank == 0 and world == 1 and not args.no_cpu_baseline else None

    write_step, decode = decode_fns(B, d, P, cascade)
    for _ in range(args.warmup):
        write_step()
        decode()
    torch.cuda.synchronize(device)
    check_device(B, "warm-up")

    evs = [(ev(), ev()) for _ in range(args.steps)]
    t_start, t_end = ev(), ev()
    clocks = Clocks(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        write_step()
        evs[i][0].record(stream)
        decode()
        evs[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    decode_ms = [a.elapsed_time(b) for a, b in evs]
    check_device(B, "the timed region")

    kv_bytes = d["kv_bytes"]
    total_ms, all_bytes = combine_ranks(total_ms, kv_bytes, world, device)
    ms_per_step = total_ms / args.steps
    value = all_bytes / (ms_per_step * 1e-3) / 1e9
    tokens_per_s = world * nseq / (ms_per_step * 1e-3)

    e2e = None if args.no_e2e else run_e2e(args, d, device, world, P)

    cpu = None
    if baseline_rows is not None:
        cpu = cpu_baseline_record(baseline_rows, d["scale"], args.cpu_seconds, d["kc"].element_size(),
                                  f"sequences {sample_seqs} of the workload (all heads)")

    peak, peak_kind = peaks()
    dec_avg_ms = statistics.mean(decode_ms)
    achieved = kv_bytes / (dec_avg_ms * 1e-3) / 1e9
    if cascade is not None:
        split = True
        n_groups = int(cascade[0].shape[0]) - 1
        # append, prefix pass (when there are groups), suffix pass, merge kernel (split suffixes only)
        launches = args.steps * (2 + (1 if n_groups else 0) + (1 if P_eff > 0 else 0) +
                                 (1 if d["pairs"] is not None else 0))
    else:
        # one launch (the KV append is fused); the merge kernel runs for 8 or more partitions, fewer are merged
        # by the decode's last CTA
        merge_kernel = split and math.ceil(d["max_len"] / P_eff) >= 8
        launches = args.steps * (1 + (1 if merge_kernel else 0) + (1 if d["pairs"] is not None else 0))
    dtype_key = str(d["kc"].dtype).replace("torch.", "")
    traffic, traffic_src = ncu_traffic((args.workload, dtype_key, P_eff, "decode" if cascade is None else "cascade"))
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {"fp8": "fp8_e4m3 cache, bf16 q", "int8": "int8 cache, bf16 q"}.get(args.kv_dtype, sh.dtype),
        "data": "synthetic",
        "config": {"workload": WORKLOADS[args.workload], "num_seqs": nseq, "num_q_heads": sh.num_q_heads,
                   "num_kv_heads": sh.num_kv_heads, "head_dim": sh.head_dim, "block_size": sh.block_size,
                   "num_blocks": int(d["kc"].shape[0]), "context_tokens": int(d["lens_host"].sum()),
                   "kv_bytes_per_step": kv_bytes, "unique_kv_bytes_per_step": d["unique_kv_bytes"],
                   "partition_tokens": P_eff,
                   "kv_dtype": dtype_key,
                   "decode": "pa_reshape_and_cache + pa_decode_cascade (shared prefixes read once per group)"
                   if cascade is not None else "pa_decode_append (KV append fused into the decode, longest sequence "
                                               "first)",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "no flush: the K/V read per step is larger than the 126 MB L2"
                   if d["unique_kv_bytes"] > 3 * 126e6 else "no flush: K/V partly L2-resident (see unique bytes)"},
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_hbm_peak": {f"of_{peak_kind}_{peak:g}": round(value / peak, 4),
                            "of_nominal_8000": round(value / 8000.0, 4)},
        "e2e": e2e,
        "gpu_launches": launches,
        "roofline": {"kernel": ("pa_decode_cascade (prefix + suffix + merge); achieved counts logical K/V bytes"
                                if cascade is not None else
                                "pa_decode" + (" (decode + partition merge)" if split else "")), "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_source": traffic_src,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback", "decode_ms_avg": round(dec_avg_ms, 5)},
        "cpu_baseline": cpu,
        "clocks": clk,
    }
    # free this workload's device memory before the per-workload records
    del d, write_step, decode
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and args.workload == "llama2_7b_mha" and args.kv_dtype == "auto" \
            and not args.cascade and not args.no_workloads:
        clocks = Clocks(device)
        clocks.start()
        line["workloads"] = run_workloads(args, device)
        line["workloads"]["clocks"] = clocks.stop()
    if rank == 0:
        print(json.dumps(line), flush=True)


def decode_record(B, d, P, steps, warmup, device, cascade=None):
    """pa_decode (or the cascade) of one workload: kernel time per launch and the
    whole step (append + decode), with the fractions of the measured peak."""
    stream = torch.cuda.current_stream(device)
    write_step, decode = decode_fns(B, d, P, cascade)
    dec, total = time_calls(write_step, decode, steps, warmup, stream)
    check_device(B, d["name"])
    peak, kind = peaks()
    ms = statistics.mean(dec)
    gbs = d["kv_bytes"] / (ms * 1e-3) / 1e9
    nseq = len(d["ids"])
    sh = d["shape"]
    P_eff = P if P >= 0 else (B.pa_decode_partition_tokens if cascade is not None
                              else B.pa_decode_ordered_partition_tokens)(nseq, sh.num_q_heads, sh.num_kv_heads,
                                                                         d["max_len"], sh.block_size)
    dtype_key = str(d["kc"].dtype).replace("torch.", "")
    traffic, src = ncu_traffic((d["name"], dtype_key, P_eff, "decode" if cascade is None else "cascade"))
    rec = {"decode_ms": round(ms, 5), "step_ms": round(total / steps, 5), "kv_bytes": d["kv_bytes"],
           "gbs": round(gbs, 1), "frac_of_measured_peak": round(gbs / peak, 4),
           "frac_of_nominal_8000": round(gbs / 8000, 4), "tokens_per_s": round(nseq / (ms * 1e-3), 1),
           "tokens_per_s_step": round(nseq / (total / steps * 1e-3), 1), "partition_tokens": P_eff,
           "kv_dtype": dtype_key, "traffic": traffic, "traffic_source": src}
    if d["unique_kv_bytes"] != d["kv_bytes"]:
        rec["unique_kv_bytes"] = d["unique_kv_bytes"]
        rec["unique_gbs"] = round(d["unique_kv_bytes"] / (ms * 1e-3) / 1e9, 1)
    return rec


def batching_trace(device, seed=0, kv_dtype="auto", num_blocks=None):
    """The continuous-batching trace, all of its steps: host block-manager work
    per step (frees, arrivals, one slot per live sequence, block tables),
    timed on the host, and each step's slots / tables / lengths uploaded for the
    device loop. Arrivals only reserve blocks: the device-filled pool stands in
    for their prompts' K/V."""
    from paged_kv_cache_361_b200 import workloads as W
    tr = W.continuous_batching(seed=seed) if num_blocks is None else \
        W.continuous_batching(seed=seed, num_blocks=num_blocks)
    sh = tr.shape
    cache, dt = make_cache(sh, tr.num_blocks, tr.free_order, kv_dtype, device)
    g = torch.Generator(device=device)
    g.manual_seed(3000 + seed)
    fill_pool(cache, tr.num_blocks, kv_dtype, g, device)
    ops = W.batching_ops(tr)
    steps, host_s = [], []
    t_host = 0.0
    pending_slots = None
    for op in ops:
        t0 = time.perf_counter()
        if op[0] == "add":
            cache.reserve(op[1], op[2])
        elif op[0] == "free":
            cache.free(op[1])
        elif op[0] == "append":
            pending_slots, pairs = cache.bm.append_slots(op[1])
            assert len(pairs) == 0
            for s in op[1]:
                cache.lens[s] += 1
        elif op[0] == "decode":
            tables, lens32, max_len = cache.decode_inputs(op[1])
            order = cache.bm.longest_first(op[1])
        t_host += time.perf_counter() - t0
        if op[0] == "decode":
            host_s.append(t_host)
            t_host = 0.0
            steps.append(dict(slots=torch.from_numpy(pending_slots).to(device),
                              tables=torch.from_numpy(tables).to(device), lens=torch.from_numpy(lens32).to(device),
                              order=torch.from_numpy(order).to(device),
                              max_len=int(max_len), tokens=int(lens32.astype(np.int64).sum()), n=len(op[1])))
    n = steps[0]["n"]
    hkv, D = sh.num_kv_heads, sh.head_dim
    io = dict(q=torch.randn((n, sh.num_q_heads, D), generator=g, device=device).to(dt),
              k=torch.randn((n, hkv, D), generator=g, device=device).to(dt),
              v=torch.randn((n, hkv, D), generator=g, device=device).to(dt),
              out=torch.empty((n, sh.num_q_heads, D), dtype=torch.float32, device=device))
    return tr, cache, steps, host_s, io


def batching_record(B, device, reps=2, kv_dtype="auto", seed=0, num_blocks=None, partition=-1):
    """Every step of the continuous-batching trace on the device, in order
    (append + pa_decode with the library's partition choice), `reps` passes
    after one untimed pass; per-step averages over the whole trace."""
    tr, cache, steps, host_s, io = batching_trace(device, seed, kv_dtype, num_blocks)
    sh = tr.shape
    eb = cache.k_cache.element_size()
    ws_bytes = max(B.pa_decode_workspace_bytes(st["n"], sh.num_q_heads, sh.num_kv_heads, sh.head_dim, st["max_len"],
                                               sh.block_size, partition) for st in steps)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)
    scale = 1.0 / math.sqrt(sh.head_dim)
    stream = torch.cuda.current_stream(device)
    kc, vc = cache.k_cache, cache.v_cache

    def one_pass(evs=None):
        for i, st in enumerate(steps):
            if evs is not None:
                evs[i][0].record(stream)
            B.pa_decode_append(io["q"], io["k"], io["v"], st["slots"], kc, vc, st["tables"], st["lens"], scale,
                               io["out"], st["max_len"], partition, ws, seq_order=st["order"])
            if evs is not None:
                evs[i][1].record(stream)

    one_pass()
    torch.cuda.synchronize()
    check_device(B, "continuous batching warm-up")
    dec, totals = [], []
    for _ in range(reps):
        evs = [(ev(), ev()) for _ in steps]
        t0, t1 = ev(), ev()
        t0.record(stream)
        one_pass(evs)
        t1.record(stream)
        torch.cuda.synchronize()
        dec.append([a.elapsed_time(b) for a, b in evs])
        totals.append(t0.elapsed_time(t1))
    check_device(B, "continuous batching")
    peak, _ = peaks()
    nsteps = len(steps)
    dec_ms = [statistics.mean(x[i] for x in dec) for i in range(nsteps)]
    kv = [st["tokens"] * sh.num_kv_heads * sh.head_dim * 2 * eb for st in steps]
    tot_dec = sum(dec_ms)
    gbs = sum(kv) / (tot_dec * 1e-3) / 1e9
    step_ms = statistics.mean(totals) / nsteps
    ntok = sum(st["n"] for st in steps)
    rec = {"steps": nsteps, "passes": reps, "decode_ms_avg": round(tot_dec / nsteps, 5),
           "decode_ms_min": round(min(dec_ms), 5), "decode_ms_max": round(max(dec_ms), 5),
           "step_ms_avg": round(step_ms, 5), "kv_bytes_avg": int(sum(kv) / nsteps),
           "gbs": round(gbs, 1), "frac_of_measured_peak": round(gbs / peak, 4),
           "frac_of_nominal_8000": round(gbs / 8000, 4), "tokens_per_s": round(ntok / (tot_dec * 1e-3), 1),
           "tokens_per_s_step": round(ntok / (step_ms * nsteps * 1e-3), 1),
           "host_block_manager_ms_avg": round(1e3 * statistics.mean(host_s), 4),
           "host_block_manager_ms_max": round(1e3 * max(host_s), 4),
           "host_note": "C++ block manager through the ctypes binding per step: frees, arrival reservations, one "
                        "slot per live sequence, block tables, longest-first dispatch order; timed on the host, "
                        "outside the device time",
           "partition_tokens": sorted({B.pa_decode_ordered_partition_tokens(st["n"], sh.num_q_heads, sh.num_kv_heads,
                                                                    st["max_len"], sh.block_size)
                                       if partition < 0 else partition for st in steps}),
           "max_parts": max(math.ceil(st["max_len"] / pt) if pt > 0 else 1
                            for st in steps for pt in [B.pa_decode_ordered_partition_tokens(
                                st["n"], sh.num_q_heads, sh.num_kv_heads, st["max_len"], sh.block_size)
                                if partition < 0 else partition]),
           "kv_dtype": str(kc.dtype).replace("torch.", "")}
    return rec, dec_ms, kv


def run_batching_line(args, rank, world, device):
    """--workload continuous_batching: the contract's line for the whole
    200-step trace (value = all steps' K/V bytes / all steps' time)."""
    from paged_kv_cache_361_b200 import binding as B
    clocks = Clocks(device)
    if world > 1:
        torch.distributed.barrier()
    clocks.start()
    rec, dec_ms, kv = batching_record(B, device, reps=max(1, args.steps // 10), kv_dtype=args.kv_dtype, seed=rank,
                                      num_blocks=args.pool_blocks)
    clk = clocks.stop()
    ms_total = rec["step_ms_avg"] * rec["steps"]
    ms_total, all_bytes = combine_ranks(ms_total, sum(kv), world, device)
    parts = rec["partition_tokens"]
    traffic, traffic_src = ncu_traffic(("continuous_batching", rec["kv_dtype"], parts[0], "decode")) \
        if len(parts) == 1 else (None, "several partition sizes in the trace")
    value = all_bytes / (ms_total * 1e-3) / 1e9
    peak, kind = peaks()
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": rec["steps"],
            "warmup": rec["steps"], "ms_per_step": rec["step_ms_avg"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": rec["kv_dtype"], "data": "synthetic",
            "config": {"workload": WORKLOADS["continuous_batching"] + (
                           f" (pool cut to {args.pool_blocks} blocks)" if args.pool_blocks else ""),
                       "passes": rec["passes"],
                       "l2": "no flush: ~0.8 GB of K/V per step against the 126 MB L2"},
            "tokens_per_s": rec["tokens_per_s_step"],
            "gpu_launches": rec["steps"] * rec["passes"] * (1 + (1 if max(parts) > 0 and rec["max_parts"] >= 8 else 0)),
            "roofline": {"kernel": "pa_decode_append (200-step average; the KV append is fused)", "bound": "hbm",
                         "achieved": rec["gbs"],
                         "peak": peak, "unit": "GB/s", "frac": rec["frac_of_measured_peak"], "traffic": traffic,
                         "traffic_source": traffic_src, "peak_source": kind},
            "batching": rec, "clocks": clk}), flush=True)


def prefill_record(B, workload, kv_dtype, steps, warmup, device, rank=0):
    """Whole-prompt prefill (pa_reshape_and_cache of every prompt token +
    pa_prefill) over a fresh paged cache: causal attention TFLOP/s with
    4 * head_dim * Hq flops per (query, visible key) pair."""
    from paged_kv_cache_361_b200 import PagedKVCache
    hq, hkv, nseq, plen = PREFILL[workload]
    D, bs = 128, 16
    nb = nseq * plen // bs + 16
    order = np.random.default_rng(rank).permutation(nb)
    if kv_dtype == "fp8":
        cache = PagedKVCache(nb, hkv, bs, D, torch.float8_e4m3fn, device, order, k_scale=4.0 / 448,
                             v_scale=4.0 / 448)
    elif kv_dtype == "int8":
        cache = PagedKVCache(nb, hkv, bs, D, torch.int8, device, order, k_scale=4.0 / 127, v_scale=4.0 / 127)
    else:
        cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, device, order)
    g = torch.Generator(device=device)
    g.manual_seed(2000 + rank)
    T = nseq * plen
    q = torch.randn(T, hq, D, generator=g, device=device).bfloat16()
    k = torch.randn(T, hkv, D, generator=g, device=device).bfloat16()
    v = torch.randn(T, hkv, D, generator=g, device=device).bfloat16()
    out = cache.prefill(list(range(nseq)), [plen] * nseq, q, k, v)
    tables, lens, max_len = cache.decode_inputs(list(range(nseq)))
    slots = torch.from_numpy(np.concatenate([cache.bm.block_table(s)[0].repeat(bs)[:plen].astype(np.int64) * bs
                                             + np.arange(plen) % bs for s in range(nseq)])).to(device)
    t = torch.from_numpy(tables).to(device)
    L = torch.from_numpy(lens).to(device)
    cu = torch.arange(0, T + 1, plen, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    pf, total = time_calls(lambda: B.pa_reshape_and_cache(k, v, slots, cache.k_cache, cache.v_cache),
                           lambda: B.pa_prefill(q, cu, cache.k_cache, cache.v_cache, t, L, D ** -0.5, out, plen,
                                                max_len), steps, warmup, stream)
    # the prompt write alone (pa_reshape_and_cache of every prompt row): HBM-bound at this size
    ap, _ = time_calls(lambda: None, lambda: B.pa_reshape_and_cache(k, v, slots, cache.k_cache, cache.v_cache),
                       steps, warmup, stream)
    check_device(B, workload)
    append_bytes = 2 * T * hkv * D * (2 + cache.k_cache.element_size())   # bf16 rows read, cache rows written
    flops = 4.0 * D * hq * nseq * plen * (plen + 1) / 2
    pf_ms = statistics.mean(pf)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    return {"workload": f"{workload}: {nseq} prompts x {plen} tokens, {hq}/{hkv} heads, D128, bs16",
            "kv_dtype": str(cache.k_cache.dtype).replace("torch.", ""), "prefill_ms": round(pf_ms, 4),
            "step_ms": round(total / steps, 4), "flops": flops,
            "tflops": round(flops / (pf_ms * 1e-3) / 1e12, 2), "peak": peak, "peak_source": src,
            "frac": round(flops / (pf_ms * 1e-3) / 1e12 / peak, 4),
            "append_ms": round(statistics.mean(ap), 4), "append_bytes": append_bytes,
            "append_gbs": round(append_bytes / (statistics.mean(ap) * 1e-3) / 1e9, 1)}


def swap_record(B, device, n_pairs=1024, reps=3):
    """Swap throughput: n_pairs blocks of the metric workload's shape (32 kv
    heads x 16 tokens x 128 dims, bf16: 128 KiB per tensor) moved out to a
    pinned host pool and back, by the pa_swap_blocks kernel (SMs reading and
    writing device-mapped host memory) and by pa_swap_blocks_copy (one
    cudaMemcpyAsync per run of consecutive ids on the copy engines; the ids
    here are scattered, so one per block)."""
    from paged_kv_cache_361_b200 import PagedKVCache
    hkv, bs, D = 32, 16, 128
    nb = 2 * n_pairs
    cache = PagedKVCache(nb, hkv, bs, D, torch.bfloat16, device)
    cache.k_cache.normal_()
    cache.v_cache.normal_()
    hk = torch.empty((n_pairs,) + tuple(cache.k_cache.shape[1:]), dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty(hk.shape, dtype=torch.bfloat16, pin_memory=True)
    rng = np.random.default_rng(7)
    dev_ids = rng.permutation(nb)[:n_pairs].astype(np.int32)
    host_ids = rng.permutation(n_pairs).astype(np.int32)
    out_pairs = np.stack([dev_ids, host_ids], 1)
    in_pairs = np.stack([host_ids, dev_ids], 1)
    dout, din = torch.from_numpy(out_pairs).to(device), torch.from_numpy(in_pairs).to(device)
    nbytes = 2 * n_pairs * hkv * bs * D * 2
    stream = torch.cuda.current_stream(device)
    rec = {"pairs": n_pairs, "bytes_each_way": nbytes}
    variants = {
        "kernel": (lambda: B.pa_swap_blocks(cache.k_cache, cache.v_cache, hk, hv, dout, True),
                   lambda: B.pa_swap_blocks(cache.k_cache, cache.v_cache, hk, hv, din, False)),
        "copy_engine": (lambda: B.pa_swap_blocks_copy(cache.k_cache, cache.v_cache, hk, hv, out_pairs, True),
                        lambda: B.pa_swap_blocks_copy(cache.k_cache, cache.v_cache, hk, hv, in_pairs, False)),
    }
    for name, (out_fn, in_fn) in variants.items():
        t_out, _ = time_calls(lambda: None, out_fn, reps, 1, stream)
        t_in, _ = time_calls(lambda: None, in_fn, reps, 1, stream)
        # host wall time of issuing the calls (the copy-engine path makes one call per run)
        t0 = time.perf_counter()
        out_fn()
        issue_ms = (time.perf_counter() - t0) * 1e3
        torch.cuda.synchronize()
        rec[name] = {"out_ms": round(statistics.mean(t_out), 4), "in_ms": round(statistics.mean(t_in), 4),
                     "out_gbs": round(nbytes / (statistics.mean(t_out) * 1e-3) / 1e9, 2),
                     "in_gbs": round(nbytes / (statistics.mean(t_in) * 1e-3) / 1e9, 2),
                     "host_issue_ms": round(issue_ms, 3)}
    # copy-on-write block copies at scale: n_pairs blocks copied within the pool
    cp = torch.from_numpy(np.stack([dev_ids, np.setdiff1d(np.arange(nb), dev_ids)[:n_pairs].astype(np.int32)],
                                   1)).to(device)
    t_cp, _ = time_calls(lambda: None, lambda: B.pa_copy_blocks(cache.k_cache, cache.v_cache, cp), reps, 1, stream)
    rec["copy_blocks"] = {"ms": round(statistics.mean(t_cp), 4), "bytes": 2 * nbytes,
                          "gbs": round(2 * nbytes / (statistics.mean(t_cp) * 1e-3) / 1e9, 1),
                          "note": "read + write bytes of the pairs' K and V blocks"}
    check_device(B, "swap")
    return rec


def run_workloads(args, device):
    """One record per workload of the pages' configurations beyond the metric
    workload (each built, timed and freed in turn)."""
    from paged_kv_cache_361_b200 import binding as B
    steps, warm = 20, 5
    rec = {}

    def release(*objs):
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    d = build_workload(0, device, "long_context_split")
    rec["long_context_split_p512"] = decode_record(B, d, 512, steps, warm, device)
    rec["long_context_split_auto"] = decode_record(B, d, -1, steps, warm, device)
    del d
    release()
    for kvd in ("fp8", "int8"):
        d = build_workload(0, device, "llama2_7b_mha", kv_dtype=kvd)
        rec[f"llama2_7b_mha_{kvd}"] = decode_record(B, d, -1, steps, warm, device)
        del d
        release()
    d = build_workload(0, device, "parallel_sampling")
    rec["parallel_sampling"] = decode_record(B, d, -1, steps, warm, device)
    rec["parallel_sampling_cascade"] = decode_record(B, d, -1, steps, warm, device, cascade_inputs(d, device))
    del d
    release()
    cb, _, _ = batching_record(B, device, reps=2)
    parts = cb["partition_tokens"]
    cb["traffic"], cb["traffic_source"] = ncu_traffic(("continuous_batching", cb["kv_dtype"], parts[0], "decode")) \
        if len(parts) == 1 else (None, "several partition sizes in the trace")
    rec["continuous_batching_200_steps"] = cb
    release()
    for wl in ("prefill_llama2_7b_mha", "prefill_gqa8"):
        r = prefill_record(B, wl, "auto", 10, 3, device)
        r["traffic"], r["traffic_source"] = ncu_traffic((wl, r["kv_dtype"], 0, "prefill"))
        rec[wl] = r
        release()
    rec["swap"] = swap_record(B, device)
    release()
    return rec


def run_e2e(args, d, device, world, P):
    """K steps through a prepared pa_step_host call (PagedKVCache.step_plan):
    per step the C++ block manager appends, the step metadata and q/k/v go host
    -> device from pinned memory, copy-on-write + append + decode run, and the
    fp32 output comes back to pinned host memory before the call returns.
    Context lengths grow by one per step. The breakdown averages the call's
    own host phase timers (pa_step_host_last_timing) and times the same bytes'
    copies alone (pinned, one stream) for the link's share."""
    from paged_kv_cache_361_b200 import binding as B
    sh = d["shape"]
    cache = d["cache"]
    ids = d["ids"]
    hq = d["q"].cpu().pin_memory()
    hk = d["k"].cpu().pin_memory()
    hv = d["v"].cpu().pin_memory()
    hout = torch.empty(d["out"].shape, dtype=torch.float32, pin_memory=True)
    eb = hq.element_size()
    plan = cache.step_plan(ids, hq, hk, hv, hout, d["scale"], partition_tokens=P,
                           max_context_len=int(max(cache.lens[s] for s in ids)) + args.warmup + args.steps + 1)
    for _ in range(args.warmup):
        plan.run()
    L0 = np.fromiter((cache.lens[s] for s in ids), dtype=np.int64, count=len(ids))
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    phases = []
    t0, t1 = ev(), ev()
    t0.record()
    for _ in range(args.steps):
        plan.run()
        phases.append(B.pa_step_host_last_timing())
    t1.record()
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1)
    # step k attends over L0 + k + 1 tokens per sequence
    n, K = len(ids), args.steps
    tokens = int(L0.sum()) * K + n * K * (K + 1) // 2
    kv_total = tokens * sh.num_kv_heads * sh.head_dim * 2 * cache.k_cache.element_size()
    nblk = int(-(-(int(L0.max()) + K) // sh.block_size))
    h2d = (hq.numel() + hk.numel() + hv.numel()) * eb + n * (8 + 8 + nblk * 4 + 4)
    d2h = hout.numel() * 4
    # the same bytes over the link alone
    dq = torch.empty(h2d, dtype=torch.uint8, device=device)
    hsrc = torch.empty(h2d, dtype=torch.uint8, pin_memory=True)
    dout = torch.empty(d2h, dtype=torch.uint8, device=device)
    hdst = torch.empty(d2h, dtype=torch.uint8, pin_memory=True)
    stream = torch.cuda.current_stream(device)
    h2d_ms, _ = time_calls(lambda: None, lambda: dq.copy_(hsrc, non_blocking=True), 10, 3, stream)
    d2h_ms, _ = time_calls(lambda: None, lambda: hdst.copy_(dout, non_blocking=True), 10, 3, stream)
    mean = lambda key: round(statistics.mean(p[key] for p in phases), 2)
    breakdown = {k: mean(k) for k in ("block_manager_us", "metadata_enqueue_us", "chains_enqueue_us", "wait_us",
                                      "total_us")}
    breakdown["chunks"] = phases[-1]["chunks"]
    breakdown["h2d_copy_alone_us"] = round(1e3 * statistics.mean(h2d_ms), 2)
    breakdown["d2h_copy_alone_us"] = round(1e3 * statistics.mean(d2h_ms), 2)
    ms, kv_total = combine_ranks(ms, kv_total, world, device)
    return {"value": round(kv_total / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(ms / args.steps, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "breakdown": breakdown,
            "api": "pa_step_host via PagedKVCache.step_plan (block manager, one metadata H2D, q/k/v H2D, "
                   "pa_copy_blocks, pa_decode_append (append fused, longest first), output D2H, stream sync)"}


PREFILL = {
    "prefill_llama2_7b_mha": (32, 32, 8, 2048),   # Hq, Hkv, sequences, prompt tokens
    "prefill_gqa8": (64, 8, 2, 8192),
}


def run_prefill(args, rank, world, device):
    """--workload prefill_*: the contract's line for whole-prompt prefill.
    --kv-dtype fp8 / int8 keeps the cache as 8-bit codes (scales 4/448, 4/127)."""
    from paged_kv_cache_361_b200 import binding as B
    clocks = Clocks(device)
    if world > 1:
        torch.distributed.barrier()
    clocks.start()
    r = prefill_record(B, args.workload, args.kv_dtype, args.steps, args.warmup, device, rank)
    clk = clocks.stop()
    ms, all_flops = combine_ranks(r["step_ms"], r["flops"], world, device)
    f8 = args.kv_dtype in ("fp8", "int8")
    traffic, traffic_src = ncu_traffic((args.workload, r["kv_dtype"], 0, "prefill"))
    if rank == 0:
        print(json.dumps({
            "metric": "paged prefill attention TFLOP/s (causal; 4*head_dim*Hq flops per visible query-key pair)",
            "value": round(all_flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": f"{'fp8_e4m3' if args.kv_dtype == 'fp8' else 'int8'} cache, bf16 q (f16 MMA)" if f8 else "bf16",
            "data": "synthetic",
            "config": {"workload": r["workload"], "kv_dtype": r["kv_dtype"], "l2": "no flush: K/V of one launch "
                       "larger than the 126 MB L2"},
            "gpu_launches": 2 * args.steps,
            "roofline": {"kernel": "pa_prefill", "bound": "tensor", "achieved": r["tflops"], "peak": r["peak"],
                         "unit": "TFLOP/s", "frac": r["frac"], "traffic": traffic, "traffic_source": traffic_src,
                         "peak_source": r["peak_source"]},
            "clocks": clk}), flush=True)


def run_reference(args, rank, world):
    """CPU oracle on this workload's shapes; each step is a bounded sample."""
    if rank != 0:
        return
    from paged_kv_cache_361_b200 import workloads as W
    w = W.llama2_7b_mha(seed=0)
    seqs = [0, 1]
    rows = [(s, w.history(s, "k"), w.history(s, "v"), w.query()[s]) for s in seqs]
    from oracle.attention import decode_attention
    bytes_per = sum(K.numel() * 2 * 2 for _, K, _, _ in rows)

    def step():
        for s, K, V, q in rows:
            decode_attention(q, K, V, w.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    ms = el * 1e3 / args.steps
    gbs = bytes_per / (ms * 1e-3) / 1e9
    sample = (f"fp64 NumPy oracle, sequences {seqs} of the workload (all 32 heads, "
              f"{bytes_per / 1e6:.1f} MB of bf16 K/V per step); host has {os.cpu_count()} cores")
    line = {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOADS["llama2_7b_mha"], "sample_seqs": seqs},
            "tokens_per_s": round(len(seqs) / (ms * 1e-3), 3),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--partition", type=int, default=-1,
                    help="partition_tokens for pa_decode (-1: library choice, -2: the workload's own)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(PREFILL), default="llama2_7b_mha")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="seconds of oracle work for each of the two CPU-baseline timings")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload records of the default run")
    ap.add_argument("--kv-dtype", choices=["auto", "fp8", "int8"], default="auto",
                    help="fp8 / int8: an 8-bit cache (e4m3 or int8 codes) with bf16 queries")
    ap.add_argument("--cascade", action="store_true",
                    help="decode through pa_decode_cascade (shared prefixes read once per group)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pool-blocks", type=int, default=None,
                    help="continuous_batching only: a smaller pool (a small case for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    from paged_kv_cache_361_b200 import build as _build
    _build.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        if args.workload in PREFILL:
            run_prefill(args, rank, world, device)
        else:
            run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
