"""PagedKVCache: a paged KV cache on one GPU, driven by the C++ block manager.

This is the public API a serving loop calls. It owns the two cache tensors
[num_blocks][num_kv_heads][block_size][head_dim], a pa_bm handle, and small
pinned staging buffers for the per-step host -> device copies of slots, tables
and lengths. All arithmetic runs in libpagedattn's kernels.

P1 = "Paged Attention：大模型推理显存优化的核心方案", P2 = "PagedAttention：操作系统级 KV
缓存虚拟内存管理".
  add_sequence  prefill write (P2 §3.2.1)
  fork          prefix sharing (P1 "跨请求的内存共享", P2 §3.4)
  append        decode-step write with copy-on-write (P2 §3.2.2 steps 1-3, §3.4)
  decode        attention over the block tables (P2 §3.2.2 step 4, §4.1)
  free          return blocks to the pool (P2 §3.3)
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import binding as B


class _Staging:
    """Host -> device upload through pinned memory. Pinned blocks come from
    torch's caching host allocator, which does not hand a block out again until
    the copies that read it have finished, so uploads never wait for the GPU."""

    def __init__(self, dtype_np, dtype_t, device):
        self.np_dtype, self.t_dtype, self.device = dtype_np, dtype_t, device

    def upload(self, arr: np.ndarray) -> torch.Tensor:
        h = torch.empty(arr.shape, dtype=self.t_dtype, pin_memory=True)
        h.numpy()[...] = arr
        return h.to(self.device, non_blocking=True)


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int,
                 dtype=torch.bfloat16, device="cuda", free_order=None, fill: float | None = None,
                 k_scale: float = 1.0, v_scale: float = 1.0):
        """dtype torch.float8_e4m3fn or torch.int8 makes an 8-bit cache with
        per-tensor scales (element = code * scale); its q/k/v inputs are bf16.
        fill sets every pool byte before use: an e4m3 cache stores the code of
        fill; an int8 cache has no NaN, so a NaN fill stores -128, the code
        quantisation never writes."""
        self.device = torch.device(device)
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = torch.empty(shape, dtype=dtype, device=self.device)
        self.v_cache = torch.empty(shape, dtype=dtype, device=self.device)
        if fill is not None:
            if dtype == torch.float8_e4m3fn:
                code = int(torch.tensor(fill, dtype=torch.float32).to(dtype).view(torch.uint8).item())
                self.k_cache.view(torch.uint8).fill_(code)
            elif dtype == torch.int8:
                self.k_cache.fill_(-128 if math.isnan(fill) else int(fill))
            else:
                self.k_cache.fill_(fill)
            self.v_cache.copy_(self.k_cache)
        if dtype in B.CODED_DTYPES:
            B.set_kv_scales(self.k_cache, self.v_cache, k_scale, v_scale)
        self.block_size = block_size
        self.bm = B.BlockManager(num_blocks, block_size, free_order)
        self.lens: dict[int, int] = {}
        self._slots = _Staging(np.int64, torch.int64, self.device)
        self._pairs = _Staging(np.int32, torch.int32, self.device)
        self._tables = _Staging(np.int32, torch.int32, self.device)
        self._lens = _Staging(np.int32, torch.int32, self.device)
        self._ws = None
        self._dev_staging = None
        self._host_staging = None

    # -- host bookkeeping + writes -------------------------------------------
    def add_sequence(self, seq_id: int, k: torch.Tensor, v: torch.Tensor) -> np.ndarray:
        n = int(k.shape[0])
        slots = self.bm.add_seq(seq_id, n)
        self.lens[seq_id] = n
        if n:
            B.pa_reshape_and_cache(k, v, self._slots.upload(slots), self.k_cache, self.v_cache)
        return slots

    def add_sequence_cached(self, seq_id: int, tokens, k: torch.Tensor, v: torch.Tensor):
        """Prefill with prefix reuse: leading whole blocks whose token prefix is
        already cached are shared (their rows are not written again); the
        other rows of k, v [n][Hkv][D] are written. Returns (slots, n_cached)."""
        slots, n_cached = self.bm.add_seq_cached(seq_id, tokens)
        n = len(slots)
        self.lens[seq_id] = n
        if n > n_cached:
            B.pa_reshape_and_cache(k[n_cached:], v[n_cached:], self._slots.upload(slots[n_cached:]),
                                   self.k_cache, self.v_cache)
        return slots, n_cached

    def reserve(self, seq_id: int, num_tokens: int) -> np.ndarray:
        """Allocate blocks for a sequence whose K/V rows the caller writes itself
        (or that are already in the pool); returns the rows' slots."""
        slots = self.bm.add_seq(seq_id, num_tokens)
        self.lens[seq_id] = num_tokens
        return slots

    def fork(self, parent: int, child: int):
        self.bm.fork(parent, child)
        self.lens[child] = self.lens[parent]

    def append(self, seq_ids, k: torch.Tensor, v: torch.Tensor):
        """One new token per listed sequence (rows of k, v in the same order).
        Returns (slots, cow_pairs) as numpy arrays."""
        slots, pairs = self.bm.append_slots(seq_ids)
        for s in seq_ids:
            self.lens[s] += 1
        if len(pairs):
            B.pa_copy_blocks(self.k_cache, self.v_cache, self._pairs.upload(pairs))
        B.pa_reshape_and_cache(k, v, self._slots.upload(slots), self.k_cache, self.v_cache)
        return slots, pairs

    def enable_swap(self, num_host_blocks: int):
        """Allocate a pinned host pool of num_host_blocks blocks (same layout)."""
        shape = (num_host_blocks,) + tuple(self.k_cache.shape[1:])
        self.host_k = torch.empty(shape, dtype=self.k_cache.dtype, pin_memory=True)
        self.host_v = torch.empty(shape, dtype=self.k_cache.dtype, pin_memory=True)
        self.bm.set_host_blocks(num_host_blocks)

    def swap_out(self, seq_id: int) -> np.ndarray:
        """Move a sequence's blocks to the host pool (P2 §五); returns the pairs."""
        pairs = self.bm.swap_out(seq_id)
        if len(pairs):
            B.pa_swap_blocks(self.k_cache, self.v_cache, self.host_k, self.host_v, self._pairs.upload(pairs), True)
        return pairs

    def swap_in(self, seq_id: int) -> np.ndarray:
        """Bring a swapped-out sequence back into fresh device blocks."""
        pairs = self.bm.swap_in(seq_id)
        if len(pairs):
            B.pa_swap_blocks(self.k_cache, self.v_cache, self.host_k, self.host_v, self._pairs.upload(pairs), False)
        return pairs

    def free(self, seq_id: int):
        self.bm.free_seq(seq_id)
        del self.lens[seq_id]

    # -- attention -------------------------------------------------------------
    def decode_inputs(self, seq_ids):
        """Host block tables [n][cap] (padded with -1) and lengths [n]."""
        max_len = max((self.lens[s] for s in seq_ids), default=0)
        cap = max(1, -(-max_len // self.block_size))
        tables, lens = self.bm.block_tables(seq_ids, cap)
        return tables, lens, max_len

    def workspace(self, nbytes: int):
        if nbytes == 0:
            return None
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    def decode(self, seq_ids, q: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None,
               partition_tokens: int = -1, longest_first: bool = True) -> torch.Tensor:
        """Decode attention for the listed sequences with queries q [n][Hq][D];
        returns fp32 [n][Hq][D]. longest_first dispatches the longest
        sequences' CTAs first (pa_bm_longest_first, pa_decode_ordered); the
        result is the same bit for bit."""
        n, hq, d = q.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        tables, lens, max_len = self.decode_inputs(seq_ids)
        if out is None:
            out = torch.empty((n, hq, d), dtype=torch.float32, device=self.device)
        hkv = self.k_cache.shape[1]
        nbytes = B.pa_decode_workspace_bytes(n, hq, hkv, d, max_len, self.block_size, partition_tokens)
        order = self._lens.upload(self.bm.longest_first(seq_ids)) if longest_first and n > 1 else None
        B.pa_decode(q, self.k_cache, self.v_cache, self._tables.upload(tables), self._lens.upload(lens), scale, out,
                    max_len, partition_tokens, self.workspace(nbytes), seq_order=order)
        return out

    def prefill(self, seq_ids, counts, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                out: torch.Tensor | None = None) -> torch.Tensor:
        """Chunked prefill: sequence seq_ids[i] takes counts[i] new tokens (a new
        sequence is created; a live one grows, with copy-on-write if it shares
        its last block). Rows of q, k, v are the new tokens of all sequences
        back to back. Writes K/V (pa_reshape_and_cache), then runs causal
        attention of the new tokens (pa_prefill); returns fp32 [T][Hq][D]."""
        counts = [int(c) for c in counts]
        T, hq, d = q.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        slots_all, pairs_all = [], []
        for s, n in zip(seq_ids, counts):
            if s in self.lens:
                sl, pr = self.bm.append_slots([s] * n)
                self.lens[s] += n
                if len(pr):
                    pairs_all.append(pr)
            else:
                sl = self.bm.add_seq(s, n)
                self.lens[s] = n
            slots_all.append(sl)
        if pairs_all:
            B.pa_copy_blocks(self.k_cache, self.v_cache, self._pairs.upload(np.concatenate(pairs_all)))
        slots = np.concatenate(slots_all) if slots_all else np.empty(0, np.int64)
        if len(slots):
            B.pa_reshape_and_cache(k, v, self._slots.upload(slots), self.k_cache, self.v_cache)
        tables, lens, max_len = self.decode_inputs(seq_ids)
        cu = np.zeros(len(counts) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(counts)
        if out is None:
            out = torch.empty((T, hq, d), dtype=torch.float32, device=self.device)
        B.pa_prefill(q, self._lens.upload(cu), self.k_cache, self.v_cache, self._tables.upload(tables),
                     self._lens.upload(lens), scale, out, max(counts, default=0), max_len)
        return out

    def shared_prefix_groups(self, seq_ids, group_rows: int):
        """Host side of the shared-prefix decode, from the C++ block manager
        (pa_bm_prefix_groups): sequences of the batch whose tables start with
        the same physical blocks form a group (at most group_rows members
        each); its prefix is the longest run of whole blocks common to all
        members, cut to a multiple of 64 tokens. Returns (offsets, members,
        prefix_tokens, seq_prefix_tokens, max_prefix)."""
        return self.bm.prefix_groups(seq_ids, group_rows, 64)

    def decode_cascade(self, seq_ids, q: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None):
        """decode() with shared prefixes (forks, prefix-cache hits) read once per
        group of sequences (pa_decode_cascade); the suffix CTAs are dispatched
        longest suffix first (pa_bm_longest_first)."""
        n, hq, d = q.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        tables, lens, max_len = self.decode_inputs(seq_ids)
        hkv = self.k_cache.shape[1]
        offs, members, prefix, seq_prefix, max_pre = self.shared_prefix_groups(seq_ids, 64 // (hq // hkv))
        order = self.bm.longest_first(seq_ids, seq_prefix)
        if out is None:
            out = torch.empty((n, hq, d), dtype=torch.float32, device=self.device)
        nbytes = B.pa_decode_cascade_workspace_bytes(n, hq, hkv, d, max_len, self.block_size, max_pre)
        ws = self.workspace(nbytes)
        empty = torch.empty(0, dtype=torch.int32, device=self.device)
        B.pa_decode_cascade(q, self.k_cache, self.v_cache, self._tables.upload(tables), self._lens.upload(lens), scale,
                            out, max_len, self._lens.upload(offs),
                            self._lens.upload(members) if len(members) else empty,
                            self._lens.upload(prefix) if len(prefix) else empty, self._lens.upload(seq_prefix),
                            int(max(np.diff(offs), default=0)), max_pre, ws, seq_order=self._lens.upload(order))
        return out

    def step_host(self, seq_ids, q_host, k_host, v_host, out_host, scale=None, partition_tokens=-1):
        """One decode step from host tensors (pinned for asynchronous copies):
        block-manager work, copies and kernels in one native call
        (pa_step_host); returns when out_host holds the fp32 result."""
        n, hq, d = q_host.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        max_len = max(self.lens[s] for s in seq_ids) + 1
        dev_b, host_b = B.pa_step_staging_bytes(n, hq, self.k_cache, self.v_cache, max_len, partition_tokens)
        if self._dev_staging is None or self._dev_staging.numel() < dev_b:
            self._dev_staging = torch.empty(dev_b * 5 // 4 + 4096, dtype=torch.uint8, device=self.device)
        if self._host_staging is None or self._host_staging.numel() < host_b:
            self._host_staging = torch.empty(host_b * 5 // 4 + 4096, dtype=torch.uint8, pin_memory=True)
        B.pa_step_host(self.bm, self.k_cache, self.v_cache, seq_ids, q_host, k_host, v_host, scale, out_host,
                       self._dev_staging, self._host_staging, partition_tokens)
        for s in seq_ids:
            self.lens[s] += 1
        return out_host

    def step_plan(self, seq_ids, q_host, k_host, v_host, out_host, scale=None, partition_tokens=-1,
                  max_context_len=None) -> "StepPlan":
        """A prepared pa_step_host call for a fixed batch and fixed host buffers:
        argument checks, staging and the C argument list are done once; each
        StepPlan.run() is one native call. Staging is sized for contexts up to
        max_context_len (default: the current maximum + 4096)."""
        return StepPlan(self, seq_ids, q_host, k_host, v_host, out_host, scale, partition_tokens, max_context_len)

    def step(self, seq_ids, q, k, v, scale=None, out=None, partition_tokens=-1):
        """One decode step: append each sequence's new K/V, then attend."""
        self.append(seq_ids, k, v)
        return self.decode(seq_ids, q, scale, out, partition_tokens)


class StepPlan:
    """See PagedKVCache.step_plan."""

    def __init__(self, cache: PagedKVCache, seq_ids, q_host, k_host, v_host, out_host, scale, partition_tokens,
                 max_context_len):
        import ctypes
        n, hq, d = q_host.shape
        self.cache = cache
        self.ids = [int(s) for s in seq_ids]
        if max_context_len is None:
            max_context_len = max(cache.lens[s] for s in self.ids) + 4096
        self.max_context_len = int(max_context_len)
        dev_b, host_b = B.pa_step_staging_bytes(n, hq, cache.k_cache, cache.v_cache, self.max_context_len,
                                                partition_tokens)
        self.dev_staging = torch.empty(dev_b, dtype=torch.uint8, device=cache.device)
        self.host_staging = torch.empty(host_b, dtype=torch.uint8, pin_memory=True)
        # validate once through the checked binding path (argument shapes, dtypes, placement)
        in_dt = B.input_dtype(cache.k_cache.dtype)
        for name, t, shape, dt in (("q_host", q_host, (n, hq, d), in_dt),
                                   ("k_host", k_host, (n, cache.k_cache.shape[1], d), in_dt),
                                   ("v_host", v_host, (n, cache.k_cache.shape[1], d), in_dt),
                                   ("out_host", out_host, (n, hq, d), torch.float32)):
            B._host(t, name, dt, shape)
        self._keep = (q_host, k_host, v_host, out_host)
        self._ids = np.ascontiguousarray(self.ids, dtype=np.int64)
        self._cache_struct = B.make_cache(cache.k_cache, cache.v_cache)
        self._args = (cache.bm._h, ctypes.byref(self._cache_struct), n, self._ids.ctypes.data_as(ctypes.c_void_p), hq,
                      q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                      float(scale if scale is not None else 1.0 / math.sqrt(d)), out_host.data_ptr(),
                      int(partition_tokens), self.dev_staging.data_ptr(), dev_b, self.host_staging.data_ptr(), host_b,
                      torch.cuda.current_stream(cache.device).cuda_stream)
        self._fn = B._lib().pa_step_host
        self.steps = 0

    def run(self):
        """One decode step; on return the output buffer holds the result."""
        if max(self.cache.lens[s] for s in self.ids) + 1 > self.max_context_len:
            raise ValueError("a sequence outgrew the plan's max_context_len")
        B._check(self._fn(*self._args), "pa_step_host")
        lens = self.cache.lens
        for s in self.ids:
            lens[s] += 1
        self.steps += 1
