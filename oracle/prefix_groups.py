"""Oracle of the shared-prefix grouping that feeds the shared-prefix decode.
TEST INFRASTRUCTURE ONLY.

P2 §3.4 (and P1 "跨请求的内存共享"): sequences that share a prefix hold the
same physical blocks in their tables. The decode can read such blocks once for
all holders; which sequences form a group is a reading, written out here as
plain Python over the block tables (a list of physical ids per sequence) and
the token counts:

  * only sequences with at least one whole block take part; they are keyed by
    the physical id of their first block, keys in order of first appearance;
  * each key's sequences, in batch order, are cut into groups of at most
    max_group rows;
  * a group's prefix is the number of leading table entries that every member
    holds identically, counted over the whole blocks of its shortest member,
    times the block size, cut down to a multiple of `align` tokens;
  * groups of one member, or whose prefix is then zero, are dropped.
Returns (offsets, members, prefix_tokens, seq_prefix_tokens) as lists.
"""
from __future__ import annotations


def prefix_groups(tables, lens, block_size: int, max_group: int, align: int):
    keys, rows_of = [], {}
    for i, (t, n) in enumerate(zip(tables, lens)):
        if n < block_size:
            continue
        k = t[0]
        if k not in rows_of:
            rows_of[k] = []
            keys.append(k)
        rows_of[k].append(i)
    offsets, members, prefix = [0], [], []
    seq_prefix = [0] * len(tables)
    for k in keys:
        rows = rows_of[k]
        for c0 in range(0, len(rows), max_group):
            grp = rows[c0:c0 + max_group]
            if len(grp) < 2:
                continue
            whole = min(lens[i] for i in grp) // block_size
            common = 0
            while common < whole and all(tables[i][common] == tables[grp[0]][common] for i in grp):
                common += 1
            ptok = common * block_size // align * align
            if ptok == 0:
                continue
            members += grp
            offsets.append(len(members))
            prefix.append(ptok)
            for i in grp:
                seq_prefix[i] = ptok
    return offsets, members, prefix, seq_prefix
