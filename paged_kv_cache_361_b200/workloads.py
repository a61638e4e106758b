"""Seeded synthetic inputs for the paged decode workloads.

This module draws random numbers and states shapes. It holds none of the
paged-attention arithmetic: no block tables, no slot numbers, no softmax. The
CPU oracle, the CUDA path, the tests and the benchmark all take their inputs
from here, so the two sides see the same values without sharing any code that
computes a result.

Page tags used in citations:
  P1 = "Paged Attention：大模型推理显存优化的核心方案" (learnblockchain.cn)
  P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理" (freeguideonline.com)
  P3 = "PagedAttention 和 vLLM" (aiunderstanding.org)

Workload recipes (none of the pages fixes these numbers beyond what is cited):
  tiny_fp32            2 sequences of 10 and 7 tokens, 4/4 heads, head_dim 64,
                       block_size 4, pool 16, fp32.  Sequence 0 is P1's worked
                       example ("Paged Attention 的工作原理": 10 tokens in
                       blocks of 4).
  llama2_7b_mha        64 sequences, lengths uniform in [128, 2048], 32/32
                       heads, head_dim 128, block_size 16 (P2 §3.1 example
                       size), pool = 1.1 x blocks needed, bf16.
  parallel_sampling    8 prompts x 1000-token shared prefix, 8 samples each,
                       tails uniform in [1, 512], 32/8 heads, head_dim 128,
                       block_size 16, bf16 (P1 "跨请求的内存共享", P2 §3.4).
  continuous_batching  pool of 200k blocks, 256 live sequences, lengths
                       lognormal(median 500, sigma 1) capped at 4096, 200
                       decode steps, finish probability 0.005 per step,
                       arrivals lognormal(median 300, sigma 1), 32/8 heads,
                       head_dim 128, block_size 16, bf16 (P2 §3.3, §4.3).
  long_context_split   4 sequences of 32768/65536/98304/131072 tokens, 64/8
                       heads, head_dim 128, block_size 32, partitions of 512
                       tokens, bf16.
All K/V/Q values are N(0, 1) drawn in fp32 and rounded to the cache dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# purpose ids for independent random streams
_LENGTHS, _FREE_ORDER, _TAILS, _FINISH, _ARRIVALS, _VALUES = 1, 2, 3, 4, 5, 6

# value kinds (keys of the value streams)
HIST_K, HIST_V, Q, NEW_K, NEW_V, PREFIX_K, PREFIX_V, TAIL_K, TAIL_V, PROMPT_K, PROMPT_V, TOKENS = range(1, 13)
_REQUESTS = 7


def _rng(seed: int, purpose: int, *keys: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), purpose, *map(int, keys)])))


def _torch_seed(seed: int, *keys: int) -> int:
    s = np.random.SeedSequence([int(seed), _VALUES, *map(int, keys)]).generate_state(2, dtype=np.uint32)
    return (int(s[0]) << 31) ^ int(s[1])


TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def normal(seed: int, keys: tuple, shape, dtype: str, device="cpu") -> torch.Tensor:
    """N(0,1) values drawn in fp32 from a generator seeded by (seed, keys), then
    rounded to `dtype` (round-to-nearest-even for bf16)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(_torch_seed(seed, *keys))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=dev)
    return x.to(TORCH_DTYPE[dtype])


@dataclass(frozen=True)
class Shape:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


@dataclass
class Workload:
    """One configuration: shapes plus every random draw it needs.

    `context_lens_old` are the sequence lengths before the measured decode step;
    the step appends one token to each, so decode attends over old + 1 tokens.
    """
    name: str
    shape: Shape
    num_blocks: int
    free_order: np.ndarray            # initial free-list order (a permutation of 0..num_blocks-1)
    context_lens_old: np.ndarray      # int64 [num_seqs]
    scale: float
    partition_tokens: int = 0         # 0: one partition per sequence
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(len(self.context_lens_old))

    @property
    def context_lens(self) -> np.ndarray:
        return self.context_lens_old + 1

    # --- values --------------------------------------------------------------
    def history(self, s: int, which: str, device="cpu") -> torch.Tensor:
        """Contiguous K or V history of sequence `s` after the step: [L_s][Hkv][D].
        The first L_s-1 rows are the prompt, the last row is the appended token."""
        L = int(self.context_lens[s])
        kind = HIST_K if which == "k" else HIST_V
        return normal(self.seed, (kind, s), (L, self.shape.num_kv_heads, self.shape.head_dim),
                      self.shape.dtype, device)

    def query(self, device="cpu") -> torch.Tensor:
        """Decode queries [num_seqs][Hq][D] in the cache dtype."""
        return normal(self.seed, (Q,), (self.num_seqs, self.shape.num_q_heads, self.shape.head_dim),
                      self.shape.dtype, device)


def _pool_for(lens_new: np.ndarray, bs: int, slack: float = 1.1) -> int:
    need = int(sum(-(-int(n) // bs) for n in lens_new))
    return int(math.ceil(slack * need))


def tiny_fp32(seed: int = 0) -> Workload:
    sh = Shape(4, 4, 64, 4, "f32")
    nb = 16
    return Workload("tiny_fp32", sh, nb, _rng(seed, _FREE_ORDER).permutation(nb).astype(np.int64),
                    np.array([10, 7], dtype=np.int64), 1.0 / math.sqrt(64), 0, seed)


def llama2_7b_mha(seed: int = 0, num_seqs: int = 64) -> Workload:
    sh = Shape(32, 32, 128, 16, "bf16")
    lens = _rng(seed, _LENGTHS).integers(128, 2048, size=num_seqs, endpoint=True).astype(np.int64)
    nb = _pool_for(lens + 1, sh.block_size)
    return Workload("llama2_7b_mha", sh, nb, _rng(seed, _FREE_ORDER).permutation(nb).astype(np.int64),
                    lens, 1.0 / math.sqrt(128), 0, seed)


def parallel_sampling(seed: int = 0, num_prompts: int = 8, num_samples: int = 8,
                      prefix_len: int = 1000, max_tail: int = 512) -> Workload:
    """Sequence id p*num_samples + j is sample j of prompt p. Its history is the
    prompt's prefix followed by its own tail; `tails[i]` counts the tail tokens
    generated before the measured step (the step appends one more)."""
    sh = Shape(32, 8, 128, 16, "bf16")
    n = num_prompts * num_samples
    tails = _rng(seed, _TAILS).integers(1, max_tail, size=n, endpoint=True).astype(np.int64)
    lens_old = prefix_len + tails
    nb = n * (-(-(prefix_len + max_tail + 1) // sh.block_size))  # no-sharing upper bound
    w = Workload("parallel_sampling", sh, nb, _rng(seed, _FREE_ORDER).permutation(nb).astype(np.int64),
                 lens_old, 1.0 / math.sqrt(128), 0, seed,
                 dict(num_prompts=num_prompts, num_samples=num_samples, prefix_len=prefix_len, tails=tails))
    return w


def prefix_values(w: Workload, p: int, which: str, device="cpu") -> torch.Tensor:
    """Shared prefix K or V of prompt p: [prefix_len][Hkv][D]."""
    kind = PREFIX_K if which == "k" else PREFIX_V
    return normal(w.seed, (kind, p), (w.extra["prefix_len"], w.shape.num_kv_heads, w.shape.head_dim),
                  w.shape.dtype, device)


def tail_values(w: Workload, s: int, which: str, device="cpu") -> torch.Tensor:
    """Own tail K or V of sample sequence s, including the measured step's token:
    [tails[s] + 1][Hkv][D]."""
    kind = TAIL_K if which == "k" else TAIL_V
    return normal(w.seed, (kind, s), (int(w.extra["tails"][s]) + 1, w.shape.num_kv_heads, w.shape.head_dim),
                  w.shape.dtype, device)


@dataclass
class BatchingTrace:
    """Random draws of the continuous-batching run.

    finish_u[step][slot] < p_finish means the sequence in batch slot `slot`
    finishes at the start of `step`; the k-th arrival of the run has prompt
    length arrival_lens[k]."""
    shape: Shape
    num_blocks: int
    free_order: np.ndarray
    initial_lens: np.ndarray
    finish_u: np.ndarray
    arrival_lens: np.ndarray
    p_finish: float
    steps: int
    seed: int

    def prompt(self, seq_id: int, length: int, which: str, device="cpu") -> torch.Tensor:
        kind = PROMPT_K if which == "k" else PROMPT_V
        return normal(self.seed, (kind, seq_id), (length, self.shape.num_kv_heads, self.shape.head_dim),
                      self.shape.dtype, device)

    def new_kv(self, step: int, which: str, n: int, device="cpu") -> torch.Tensor:
        kind = NEW_K if which == "k" else NEW_V
        return normal(self.seed, (kind, step), (n, self.shape.num_kv_heads, self.shape.head_dim),
                      self.shape.dtype, device)

    def query(self, step: int, n: int, device="cpu") -> torch.Tensor:
        return normal(self.seed, (Q, step), (n, self.shape.num_q_heads, self.shape.head_dim),
                      self.shape.dtype, device)


def _lognormal_lengths(rng: np.random.Generator, median: float, sigma: float, n: int, cap: int) -> np.ndarray:
    x = rng.lognormal(mean=math.log(median), sigma=sigma, size=n)
    return np.clip(np.rint(x), 1, cap).astype(np.int64)


def continuous_batching(seed: int = 0, num_live: int = 256, steps: int = 200, num_blocks: int = 200_000,
                        p_finish: float = 0.005) -> BatchingTrace:
    sh = Shape(32, 8, 128, 16, "bf16")
    init = _lognormal_lengths(_rng(seed, _LENGTHS), 500.0, 1.0, num_live, 4096)
    fin = _rng(seed, _FINISH).random((steps, num_live))
    arr = _lognormal_lengths(_rng(seed, _ARRIVALS), 300.0, 1.0, steps * num_live, 4096)
    order = _rng(seed, _FREE_ORDER).permutation(num_blocks).astype(np.int64)
    return BatchingTrace(sh, num_blocks, order, init, fin, arr, p_finish, steps, seed)


def long_context_split(seed: int = 0) -> Workload:
    sh = Shape(64, 8, 128, 32, "bf16")
    lens = np.array([32768, 65536, 98304, 131072], dtype=np.int64)
    nb = _pool_for(lens + 1, sh.block_size)
    return Workload("long_context_split", sh, nb, _rng(seed, _FREE_ORDER).permutation(nb).astype(np.int64),
                    lens, 1.0 / math.sqrt(128), 512, seed)


def random_small(seed: int, num_seqs: int, shape: Shape, max_len: int, slack_blocks: int = 3) -> Workload:
    """A small random case for fuzzing: lengths uniform in [0, max_len - 1] before
    the step, pool sized to the blocks needed plus `slack_blocks`."""
    lens = _rng(seed, _LENGTHS).integers(0, max_len, size=num_seqs).astype(np.int64)
    nb = int(sum(-(-int(n + 1) // shape.block_size) for n in lens)) + slack_blocks
    return Workload(f"random_small_{seed}", shape, nb, _rng(seed, _FREE_ORDER).permutation(nb).astype(np.int64),
                    lens, 1.0 / math.sqrt(shape.head_dim), 0, seed)


# --- operation scripts ---------------------------------------------------------
# Each recipe is a list of block-manager / kernel operations in a fixed order.
# Both the oracle and the CUDA path replay the same list with their own code.
# Values are produced on demand by the `src` callables: src(which, device) for
# K ("k") or V ("v") rows, src(device) for queries.
#
#   ("add", seq_id, num_tokens, src)   prefill: allocate, then write num_tokens rows
#   ("fork", parent, child)            child shares parent's blocks
#   ("append", [seq_ids], src)         one new token per listed sequence, in order
#   ("free", seq_id)                   sequence finished
#   ("decode", [seq_ids], qsrc)        one decode step over the listed sequences


def simple_ops(w: Workload) -> list:
    """Prefill every sequence in index order, append one token to each, decode."""
    ops = []
    for s in range(w.num_seqs):
        n = int(w.context_lens_old[s])
        ops.append(("add", s, n, (lambda which, device="cpu", s=s, n=n: w.history(s, which, device)[:n])))
    ops.append(("append", list(range(w.num_seqs)),
                lambda which, device="cpu": torch.stack(
                    [w.history(s, which, device)[int(w.context_lens_old[s])] for s in range(w.num_seqs)])))
    ops.append(("decode", list(range(w.num_seqs)), lambda device="cpu": w.query(device)))
    return ops


def sampling_ops(w: Workload, batch_tail_steps: bool = False) -> list:
    """Parallel sampling: sample 0 of each prompt is prefilled with the prefix,
    samples 1..n-1 fork from it, tails are generated in lockstep (one token per
    unfinished sample per step, samples in id order), then the measured step
    appends one token to every sample and decodes all of them.

    With batch_tail_steps, lockstep steps 2..max are merged into one append
    list (same order of slot assignment, one write)."""
    P, S, pre = w.extra["num_prompts"], w.extra["num_samples"], w.extra["prefix_len"]
    tails = w.extra["tails"]
    ops = []
    for p in range(P):
        ops.append(("add", p * S, pre, (lambda which, device="cpu", p=p: prefix_values(w, p, which, device))))
        for j in range(1, S):
            ops.append(("fork", p * S, p * S + j))
    max_tail = int(tails.max())

    def step_src(ids, tau):
        return lambda which, device="cpu": torch.stack([tail_values(w, s, which, device)[tau - 1] for s in ids])

    pending_ids, pending_taus = [], []
    for tau in range(1, max_tail + 1):
        ids = [s for s in range(P * S) if int(tails[s]) >= tau]
        if batch_tail_steps and tau >= 2:
            pending_ids += ids
            pending_taus += [tau] * len(ids)
            continue
        ops.append(("append", ids, step_src(ids, tau)))
    if pending_ids:
        def merged(which, device="cpu", ids=tuple(pending_ids), taus=tuple(pending_taus)):
            cache = {}
            rows = []
            for s, t in zip(ids, taus):
                if s not in cache:
                    cache[s] = tail_values(w, s, which, device)
                rows.append(cache[s][t - 1])
            return torch.stack(rows)
        ops.append(("append", list(pending_ids), merged))
    all_ids = list(range(P * S))
    ops.append(("append", all_ids, lambda which, device="cpu": torch.stack(
        [tail_values(w, s, which, device)[int(tails[s])] for s in all_ids])))
    ops.append(("decode", all_ids, lambda device="cpu": w.query(device)))
    return ops


def sampling_history(w: Workload, s: int, which: str, device="cpu") -> torch.Tensor:
    """Contiguous history of sample s after the measured step: prefix ++ tail."""
    p = s // w.extra["num_samples"]
    return torch.cat([prefix_values(w, p, which, device), tail_values(w, s, which, device)])


def batching_ops(tr: BatchingTrace, steps: int | None = None) -> list:
    """Continuous batching: the initial sequences (ids 0..num_live-1) are
    prefilled in slot order. At each step, the sequences whose finish draw is
    below p_finish are freed and each is replaced, in the same batch slot and in
    slot order, by a new arrival (fresh id, prefilled); then every live sequence
    appends one token in slot order and the batch decodes."""
    steps = tr.steps if steps is None else steps
    live = list(range(len(tr.initial_lens)))
    next_id = len(live)
    ops = []
    for s in live:
        n = int(tr.initial_lens[s])
        ops.append(("add", s, n, (lambda which, device="cpu", s=s, n=n: tr.prompt(s, n, which, device))))
    k_arr = 0
    for step in range(steps):
        for slot in range(len(live)):
            if tr.finish_u[step, slot] < tr.p_finish:
                ops.append(("free", live[slot]))
                n = int(tr.arrival_lens[k_arr])
                k_arr += 1
                sid = next_id
                next_id += 1
                live[slot] = sid
                ops.append(("add", sid, n, (lambda which, device="cpu", sid=sid, n=n: tr.prompt(sid, n, which, device))))
        ids = list(live)
        ops.append(("append", ids, (lambda which, device="cpu", step=step, n=len(ids): tr.new_kv(step, which, n, device))))
        ops.append(("decode", ids, (lambda device="cpu", step=step, n=len(ids): tr.query(step, n, device))))
    return ops


@dataclass
class PrefixTrace:
    """Requests that start with one of a few shared system prompts.

    Request r uses system prompt sys_of[r] (its tokens sys_tokens[k], K/V rows
    drawn per (system prompt, position), so every request that shares it sees
    the same rows) followed by its own tail of tail_lens[r] tokens. Requests
    arrive in order; at most `live` run at once; when the batch is full the
    oldest request finishes first (FIFO), before each decode step every live
    request appends one token."""
    shape: Shape
    num_blocks: int
    free_order: np.ndarray
    sys_tokens: list
    sys_of: np.ndarray
    tail_lens: np.ndarray
    live: int
    seed: int

    def request_tokens(self, r: int) -> np.ndarray:
        tail = _rng(self.seed, _REQUESTS, r).integers(1000, 32000, size=int(self.tail_lens[r]))
        return np.concatenate([self.sys_tokens[int(self.sys_of[r])], tail]).astype(np.int32)

    def rows(self, r: int, which: str, device="cpu") -> torch.Tensor:
        """K or V rows of request r's prompt: system part then tail."""
        k = int(self.sys_of[r])
        sys_n = len(self.sys_tokens[k])
        a = normal(self.seed, (PREFIX_K if which == "k" else PREFIX_V, k),
                   (sys_n, self.shape.num_kv_heads, self.shape.head_dim), self.shape.dtype, device)
        b = normal(self.seed, (TAIL_K if which == "k" else TAIL_V, r),
                   (int(self.tail_lens[r]), self.shape.num_kv_heads, self.shape.head_dim), self.shape.dtype, device)
        return torch.cat([a, b])


def prefix_caching(seed: int = 0, num_sys: int = 4, sys_len: int = 700, num_requests: int = 48, live: int = 16,
                   num_blocks: int = 500, block_size: int = 16, head_dim: int = 128) -> PrefixTrace:
    """A small pool (num_blocks) so that cached blocks get evicted."""
    sh = Shape(32, 8, head_dim, block_size, "bf16")
    rng = _rng(seed, _TOKENS_PURPOSE)
    sys_tokens = [rng.integers(1000, 32000, size=sys_len - 37 * k).astype(np.int32) for k in range(num_sys)]
    sys_of = _rng(seed, _LENGTHS, 11).integers(0, num_sys, size=num_requests)
    tails = _rng(seed, _TAILS, 11).integers(1, 257, size=num_requests)
    order = _rng(seed, _FREE_ORDER).permutation(num_blocks).astype(np.int64)
    return PrefixTrace(sh, num_blocks, order, sys_tokens, sys_of, tails, live, seed)


_TOKENS_PURPOSE = 8


def prefix_ops(tr: PrefixTrace, decode_every: int = 4) -> list:
    """Requests arrive one by one ("add_cached"); when `live` are running the
    oldest finishes first; every request appends one token per step and the
    batch decodes every `decode_every` arrivals and at the end."""
    ops, live = [], []
    for r in range(len(tr.sys_of)):
        if len(live) == tr.live:
            ops.append(("free", live.pop(0)))
        toks = tr.request_tokens(r)
        ops.append(("add_cached", r, toks, (lambda which, device="cpu", r=r: tr.rows(r, which, device))))
        live.append(r)
        if r % decode_every == decode_every - 1 or r == len(tr.sys_of) - 1:
            ids = list(live)
            ops.append(("append", ids, (lambda which, device="cpu", r=r, n=len(ids): normal(
                tr.seed, (NEW_K if which == "k" else NEW_V, r), (n, tr.shape.num_kv_heads, tr.shape.head_dim),
                tr.shape.dtype, device))))
            ops.append(("decode", ids, (lambda device="cpu", r=r, n=len(ids): normal(
                tr.seed, (Q, r), (n, tr.shape.num_q_heads, tr.shape.head_dim), tr.shape.dtype, device))))
    return ops
