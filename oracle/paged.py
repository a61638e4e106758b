"""Oracle for the paged cache's data movement.

Pool layout (a reading: the pages fix none): K and V pools are each
[num_blocks][num_kv_heads][block_size][head_dim]; token t of a sequence lives at
physical block table[t // block_size], offset t % block_size (P2 §2.3 and §五:
the table gives the physical block, the offset within it gives the token).

  scatter      P2 §3.2.2 step 3 ("write the new K, V at the block position"),
               and P2 §3.2.1 for a prompt; slot -1 is skipped.
  gather       P2 §3.2.2 step 4 and §4.1: attention visits every logical block
               through the table.
  copy_blocks  P2 §3.4: the copy made before writing into a shared block.

Pools are torch CPU tensors so that bf16 values are held exactly; every
operation here is a bit copy.
"""
from __future__ import annotations

import torch


def new_pool(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int, dtype,
             fill: float = float("nan")) -> torch.Tensor:
    return torch.full((num_blocks, num_kv_heads, block_size, head_dim), fill, dtype=dtype)


def scatter(pool: torch.Tensor, rows: torch.Tensor, slots) -> None:
    """pool[slot // bs, :, slot % bs, :] = rows[i] for each i with slot != -1."""
    bs = pool.shape[2]
    for i, slot in enumerate(slots):
        slot = int(slot)
        if slot == -1:
            continue
        pool[slot // bs, :, slot % bs, :] = rows[i]


def gather(pool: torch.Tensor, table, length: int) -> torch.Tensor:
    """Rows of tokens 0..length-1 in logical order: [length][Hkv][D]."""
    bs = pool.shape[2]
    out = torch.empty((length, pool.shape[1], pool.shape[3]), dtype=pool.dtype)
    for t in range(length):
        out[t] = pool[int(table[t // bs]), :, t % bs, :]
    return out


def copy_blocks(pool: torch.Tensor, pairs) -> None:
    """pool[dst] = pool[src], pair by pair in the given order."""
    for src, dst in pairs:
        pool[int(dst)] = pool[int(src)].clone()
