"""CPU oracle for paged decode attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package. The library (paged_kv_cache_361_b200) never does, and it shares
no code with it: the oracle has its own block manager, its own scatter/gather
and its own attention, all plain Python / NumPy in fp64 (PyTorch CPU tensors are
used only to hold bf16 values and to copy bits).

Page tags used in citations:
  P1 = "Paged Attention：大模型推理显存优化的核心方案" (learnblockchain.cn)
  P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理" (freeguideonline.com)
  P3 = "PagedAttention 和 vLLM" (aiunderstanding.org)

Modules and what pins each one (tests/test_oracle_*.py):
  block_manager  free list, refcounts, block-table growth, copy-on-write.
                 Pinned by P1's worked example (10 tokens in blocks of 4, the
                 block table 0->5, 1->12, 2->3; tests/golden), the contiguous
                 preallocation waste of the same example, and invariants
                 (refcounts equal table references, no block both free and
                 used, waste only in last blocks).
  paged          slot scatter, block-table gather, block copy.  Pinned by
                 gather == contiguous history bitwise, under any permutation
                 of physical ids and any block size.
  attention      softmax(scale * q K^T) V per query head, GQA by contiguous
                 groups, and the partitioned form with its log-sum-exp merge.
                 Pinned by closed forms (one token returns v0; equal keys or
                 q = 0 return the mean of V; two tokens reduce to the logistic
                 function; a key built to score ln 3 higher weights 3:1), the
                 head-to-group map, shift invariance, and a 50-digit mpmath
                 brute force on tiny inputs.
  prefix_groups  which batch sequences share leading physical blocks and how
                 many tokens of them (the host side of the shared-prefix
                 decode). Pinned by hand-worked cases (forks of one prompt,
                 a copy-on-write split inside the prefix, lone sequences,
                 group-size cuts, the alignment cut) in
                 tests/test_oracle_prefix_groups.py.
  replay         replays an operation script (paged_kv_cache_361_b200.workloads)
                 on the oracle's block manager and a contiguous per-sequence
                 history (the "traditional" layout of P1 and P2 §1.2).
No function here is "parity unpinned".
"""
