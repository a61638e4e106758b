#!/usr/bin/env python
"""Decode-step benchmark of libpagedattn on the Llama-2-7B-shaped workload.

Workload: 64 sequences, context lengths uniform in [128, 2048] before the step
(one token appended, then decode), 32 query heads = 32 kv heads, head_dim 128,
block_size 16, bf16 cache, pool = 1.1 x blocks needed with ids in a seeded
shuffle, Q/K/V ~ N(0, 1). One step = the whole hot path for one batch: KV
append (pa_reshape_and_cache) + decode attention (pa_decode, split into
partitions with its log-sum-exp merge when the library chooses to).

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

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# dominant kernel, from an ncu capture of
#   python bench.py --steps 3 --warmup 3 --no-e2e --no-cpu-baseline
# (profiles/decode_simt_llama2_7b_mha.md), keyed by (workload, cache dtype,
# partition tokens). Configurations without a capture of the current kernel
# report null.
NCU_TRAFFIC = {("llama2_7b_mha", "bfloat16", 0): 1_082_858_240}


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
    "continuous_batching": "continuous_batching_decode: 256 live seqs, ctx lognormal(500,1) capped 4096, first step "
                           "of the trace, 200k-block pool, 32/8 heads, D128, bs16, bf16",
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
    from paged_kv_cache_361_b200 import PagedKVCache
    from paged_kv_cache_361_b200 import workloads as W
    sh, nb, order, scale, part, ops = workload_ops(name, seed)
    dt = W.TORCH_DTYPE[sh.dtype]
    cache_dt = {"fp8": torch.float8_e4m3fn, "int8": torch.int8}.get(kv_dtype, dt)
    sc = 4.0 / 127 if kv_dtype == "int8" else 1.0
    cache = PagedKVCache(nb, sh.num_kv_heads, sh.block_size, sh.head_dim, cache_dt, device, order, k_scale=sc,
                         v_scale=sc)
    g = torch.Generator(device=device)
    g.manual_seed(1000 + seed)
    for t in (cache.k_cache, cache.v_cache):
        for i in range(0, nb, 1024):   # chunked to bound the fp32 temporary
            if kv_dtype == "int8":
                t[i:i + 1024] = torch.randint(-127, 128, t[i:i + 1024].shape, generator=g, device=device,
                                              dtype=torch.int8)
            else:
                t[i:i + 1024] = torch.randn(t[i:i + 1024].shape, generator=g, device=device).to(cache_dt)
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
    done once, before timing): sequences whose tables start with the same
    blocks share their common prefix."""
    from paged_kv_cache_361_b200 import binding as B
    cache, sh = d["cache"], d["shape"]
    tables = d["tables"].cpu().numpy()
    lens = d["lens"].cpu().numpy()
    offs, members, prefix, seq_prefix = cache.shared_prefix_groups(d["ids"], tables, lens,
                                                                   64 // sh.group)
    max_pre = int(prefix.max()) if len(prefix) else 0
    nbytes = B.pa_decode_cascade_workspace_bytes(len(d["ids"]), sh.num_q_heads, sh.num_kv_heads, sh.head_dim,
                                                 d["max_len"], sh.block_size, max_pre)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    return (t(offs), t(members), t(prefix), t(seq_prefix), int(max(np.diff(offs), default=0)), max_pre, ws)


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


# --- arms --------------------------------------------------------------------------

def run_ours(args, rank, world, device):
    from paged_kv_cache_361_b200 import binding as B
    d = build_workload(seed=rank, device=device, name=args.workload, kv_dtype=args.kv_dtype)
    sh = d["shape"]
    nseq = len(d["ids"])
    cascade = None
    if args.cascade:
        cascade = cascade_inputs(d, device)
    P = args.partition if args.partition != -2 else d["part"]
    ws_bytes = B.pa_decode_workspace_bytes(nseq, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, d["max_len"],
                                           sh.block_size, P)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device) if ws_bytes else None
    P_eff = P if P >= 0 else B.pa_decode_partition_tokens(nseq, sh.num_q_heads, sh.num_kv_heads, d["max_len"],
                                                          sh.block_size)
    split = P_eff > 0 and math.ceil(d["max_len"] / P_eff) > 1
    stream = torch.cuda.current_stream(device)

    sample_seqs = [0, 1, 2, 3] if args.workload == "llama2_7b_mha" else [0]
    baseline_rows = sample_rows(d, sample_seqs) if rank == 0 and world == 1 and not args.no_cpu_baseline else None

    def write_step():
        if d["pairs"] is not None:
            B.pa_copy_blocks(d["kc"], d["vc"], d["pairs"])
        B.pa_reshape_and_cache(d["k"], d["v"], d["slots"], d["kc"], d["vc"])

    def decode():
        if cascade is not None:
            B.pa_decode_cascade(d["q"], d["kc"], d["vc"], d["tables"], d["lens"], d["scale"], d["out"], d["max_len"],
                                *cascade)
            return
        B.pa_decode(d["q"], d["kc"], d["vc"], d["tables"], d["lens"], d["scale"], d["out"], d["max_len"], P, ws)

    for _ in range(args.warmup):
        write_step()
        decode()
    torch.cuda.synchronize(device)
    st, info = B.pa_get_device_error()
    if st != B.PA_OK:
        raise RuntimeError(f"device error {st} ({info}) during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        write_step()
        ev[i][0].record(stream)
        decode()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    decode_ms = [a.elapsed_time(b) for a, b in ev]
    st, info = B.pa_get_device_error()
    if st != B.PA_OK:
        raise RuntimeError(f"device error {st} ({info}) in the timed region")

    kv_bytes = d["kv_bytes"]
    total_ms, all_bytes = combine_ranks(total_ms, kv_bytes, world, device)
    ms_per_step = total_ms / args.steps
    value = all_bytes / (ms_per_step * 1e-3) / 1e9
    tokens_per_s = world * nseq / (ms_per_step * 1e-3)

    e2e = None if args.no_e2e else run_e2e(args, d, device, world, P)

    cpu = None
    if baseline_rows is not None:
        gbs, el, n = time_oracle(baseline_rows, d["scale"], args.cpu_seconds, d["kc"].element_size())
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"fp64 NumPy oracle over sequences {sample_seqs} of the workload (all heads), repeated "
                         f"for {el:.1f} s ({n} sequence passes); host has {os.cpu_count()} cores"}

    peak, peak_kind = peaks()
    dec_avg_ms = statistics.mean(decode_ms)
    achieved = kv_bytes / (dec_avg_ms * 1e-3) / 1e9
    if cascade is not None:
        split = True
        n_groups = int(cascade[0].shape[0]) - 1
        launches = args.steps * (1 + (1 if n_groups else 0) + 2 + (1 if d["pairs"] is not None else 0))
    else:
        launches = args.steps * (2 + (1 if split else 0) + (1 if d["pairs"] is not None else 0))
    if rank == 0:
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
                       "kv_dtype": str(d["kc"].dtype).replace("torch.", ""),
                       "decode": "pa_decode_cascade (shared prefixes read once per group)" if cascade is not None
                       else "pa_decode",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                       "l2": "no flush: the K/V read per step is larger than the 126 MB L2"
                       if d["unique_kv_bytes"] > 3 * 126e6 else "no flush: K/V partly L2-resident (see unique bytes)"},
            "tokens_per_s": round(tokens_per_s, 1),
            "pct_of_hbm_peak": {"of_measured_6540": round(value / peak, 4), "of_nominal_8000": round(value / 8000.0, 4)},
            "e2e": e2e,
            "gpu_launches": launches,
            "roofline": {"kernel": ("pa_decode_cascade (prefix + suffix + merge); achieved counts logical K/V bytes"
                                    if cascade is not None else
                                    "pa_decode" + (" (decode + partition merge)" if split else "")), "bound": "hbm",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": None if cascade is not None else NCU_TRAFFIC.get(
                             (args.workload, str(d["kc"].dtype).replace("torch.", ""), P_eff)),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                         else "fallback", "decode_ms_avg": round(dec_avg_ms, 5)},
            "cpu_baseline": cpu,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def run_e2e(args, d, device, world, P):
    """K steps through a prepared pa_step_host call (PagedKVCache.step_plan):
    per step the C++ block manager appends, the step metadata and q/k/v go host
    -> device from pinned memory, copy-on-write + append + decode run, and the
    fp32 output comes back to pinned host memory before the call returns.
    Context lengths grow by one per step."""
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
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        plan.run()
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
    ms, kv_total = combine_ranks(ms, kv_total, world, device)
    return {"value": round(kv_total / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(ms / args.steps, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "pa_step_host via PagedKVCache.step_plan (block manager, one metadata H2D, q/k/v H2D, "
                   "pa_copy_blocks, pa_reshape_and_cache, pa_decode, output D2H, stream sync)"}


PREFILL = {
    "prefill_llama2_7b_mha": (32, 32, 8, 2048),   # Hq, Hkv, sequences, prompt tokens
    "prefill_gqa8": (64, 8, 2, 8192),
}


def run_prefill(args, rank, world, device):
    """Whole-prompt prefill (pa_reshape_and_cache of every prompt token +
    pa_prefill) over a fresh paged cache; metric: causal attention TFLOP/s with
    4 * head_dim * Hq flops per (query, visible key) pair. --kv-dtype fp8 keeps
    the cache as e4m3 codes (per-tensor scales 4/448: N(0, 1) rows use the
    code range)."""
    from paged_kv_cache_361_b200 import PagedKVCache, binding as B
    hq, hkv, nseq, plen = PREFILL[args.workload]
    D, bs = 128, 16
    nb = nseq * plen // bs + 16
    order = np.random.default_rng(rank).permutation(nb)
    f8 = args.kv_dtype in ("fp8", "int8")
    if args.kv_dtype == "fp8":
        cache = PagedKVCache(nb, hkv, bs, D, torch.float8_e4m3fn, device, order, k_scale=4.0 / 448,
                             v_scale=4.0 / 448)
    elif args.kv_dtype == "int8":
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

    def step():
        B.pa_reshape_and_cache(k, v, slots, cache.k_cache, cache.v_cache)
        B.pa_prefill(q, cu, cache.k_cache, cache.v_cache, t, L, D ** -0.5, out, plen, max_len)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    e0.record(stream)
    for i in range(args.steps):
        B.pa_reshape_and_cache(k, v, slots, cache.k_cache, cache.v_cache)
        ev[i][0].record(stream)
        B.pa_prefill(q, cu, cache.k_cache, cache.v_cache, t, L, D ** -0.5, out, plen, max_len)
        ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    st, info = B.pa_get_device_error()
    if st != B.PA_OK:
        raise RuntimeError(f"device error {st} ({info})")
    ms = e0.elapsed_time(e1) / args.steps
    pf_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = 4.0 * D * hq * nseq * plen * (plen + 1) / 2
    ms, all_flops = combine_ranks(ms, flops, world, device)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    if rank == 0:
        print(json.dumps({
            "metric": "paged prefill attention TFLOP/s (causal; 4*head_dim*Hq flops per visible query-key pair)",
            "value": round(all_flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": f"{'fp8_e4m3' if args.kv_dtype == 'fp8' else 'int8'} cache, bf16 q (f16 MMA)" if f8 else "bf16",
            "data": "synthetic",
            "config": {"workload": f"{args.workload}: {nseq} prompts x {plen} tokens, {hq}/{hkv} heads, D128, bs16",
                       "kv_dtype": str(cache.k_cache.dtype).replace("torch.", ""),
                       "l2": "no flush: K/V of one launch "
                             + f"{2 * T * hkv * D * (1 if f8 else 2) / 1e6:.0f} MB"},
            "gpu_launches": 2 * args.steps,
            "roofline": {"kernel": "pa_prefill", "bound": "tensor", "achieved": round(flops / (pf_ms * 1e-3) / 1e12, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(flops / (pf_ms * 1e-3) / 1e12 / peak, 4),
                         "traffic": None, "peak_source": src,
                         "note": ("tcgen05.mma (M 128) with TMEM accumulators; K/V codes widened to f16 in "
                                  "shared memory, one f16 P V MMA per k-step") if f8 else
                                 ("tcgen05.mma (M 128) with TMEM accumulators; P split into two bf16 MMAs "
                                  "(1.5x the algorithmic MMA work)")},
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
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--kv-dtype", choices=["auto", "fp8", "int8"], default="auto",
                    help="fp8 / int8: an 8-bit cache (e4m3 or int8 codes) with bf16 queries")
    ap.add_argument("--cascade", action="store_true",
                    help="decode through pa_decode_cascade (shared prefixes read once per group)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
