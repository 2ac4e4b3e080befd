"""Shared-prefix groups of a decode batch. Test infrastructure only.

Prefix sharing is described in "PagedAttention: treat the cache like virtual
memory" (KV-Cache Management and PagedAttention: many requests that start with
the same system prompt point their block tables at the same physical blocks),
in "Shared System Prompts & Prefix Caching" (PagedAttention and KV Cache
Management) and in "RadixAttention — reuse a shared prefix" (the third page:
a shared beginning is stored once, only the suffix is per request). A block
id that appears in several rows of the block tables therefore holds the same
K/V for all of them, and attention over those rows can read it once.

The grouping below is the plain definition the library's host helper must
reproduce bit for bit:

  * A row (batch position) is a candidate when its first block is full
    (context length >= B); candidates are grouped by that first block id.
  * A group is kept when it has at least `min_members` rows. Its shared
    prefix is the longest run of leading table columns j whose entry is the
    same block in every member and is full in every member ((j + 1) * B <= L).
  * Kept groups are listed in the order of their lowest row; members in
    ascending row order. Rows outside kept groups get prefix_blocks 0.

Outputs: group_start [G + 1], members [M] (rows), prefix_blocks [S].
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def prefix_groups(tables: np.ndarray, lens: Sequence[int], block_size: int,
                  min_members: int = 2) -> Tuple[List[int], List[int], List[int]]:
    tables = np.asarray(tables)
    S = len(lens)
    B = block_size
    by_first = {}
    order = []
    for row in range(S):
        if int(lens[row]) >= B:
            key = int(tables[row, 0])
            if key not in by_first:
                by_first[key] = []
                order.append(key)
            by_first[key].append(row)
    group_start, members = [0], []
    prefix_blocks = [0] * S
    for key in order:
        rows = by_first[key]
        if len(rows) < min_members:
            continue
        n = 0
        while True:
            j = n
            full = all((j + 1) * B <= int(lens[r]) for r in rows)
            if not full or j >= tables.shape[1]:
                break
            if any(int(tables[r, j]) != int(tables[rows[0], j]) for r in rows):
                break
            n += 1
        members.extend(rows)
        group_start.append(len(members))
        for r in rows:
            prefix_blocks[r] = n
    return group_start, members, prefix_blocks
