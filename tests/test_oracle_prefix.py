"""Pins of the shared-prefix grouping (oracle/prefix.py).

Prefix sharing: "PagedAttention: treat the cache like virtual memory"
(KV-Cache Management and PagedAttention), "Shared System Prompts & Prefix
Caching" (PagedAttention and KV Cache Management), "RadixAttention — reuse a
shared prefix" (the third page).
"""
import itertools

import numpy as np
import pytest

import workloads as W
from oracle.allocator import BlockAllocator
from oracle.prefix import prefix_groups


def _table(rows, width):
    t = np.full((len(rows), width), -1, dtype=np.int64)
    for i, r in enumerate(rows):
        t[i, :len(r)] = r
    return t


# B = 4. Worked by hand:
#   rows 0, 1, 2 start with block 7 (full in all three). Column 1 holds block 3
#   in rows 0 and 1 but block 8 in row 2, and row 2 has only 6 tokens (its
#   second block is not full either), so the group shares 1 block.
#   rows 3, 4 start with blocks 2, 4, both full in both (8 <= 8, 8 <= 11);
#   column 2 is not full in row 3, so they share 2 blocks.
#   row 5's first block is not full (3 tokens): no candidate.
#   row 6 is the only row starting with block 1: a group of one is dropped.
HAND_TABLES = _table([[7, 3, 9], [7, 3, 5], [7, 8], [2, 4], [2, 4, 6], [1], [1, 0]], 4)
HAND_LENS = [10, 12, 6, 8, 11, 3, 5]


def test_hand_worked_case():
    gs, mem, pb = prefix_groups(HAND_TABLES, HAND_LENS, 4)
    assert gs == [0, 3, 5]
    assert mem == [0, 1, 2, 3, 4]
    assert pb == [1, 1, 1, 2, 2, 0, 0]


def test_min_members_drops_small_groups():
    gs, mem, pb = prefix_groups(HAND_TABLES, HAND_LENS, 4, min_members=3)
    assert gs == [0, 3] and mem == [0, 1, 2] and pb == [1, 1, 1, 0, 0, 0, 0]


def test_boundary_fullness():
    # 8 tokens at B = 4: both blocks full; 7 tokens: the second is not.
    t = _table([[5, 6], [5, 6]], 2)
    assert prefix_groups(t, [8, 8], 4)[2] == [2, 2]
    assert prefix_groups(t, [8, 7], 4)[2] == [1, 1]
    assert prefix_groups(t, [3, 8], 4) == ([0], [], [0, 0])


def _prefix_layout(spec):
    sc = W.prefix_script(spec)
    a = BlockAllocator(sc.num_blocks, spec.block_size, sc.free_order)
    a.run(sc.setup)
    for r in sc.step_appends:
        a.append_slot(r)
    width = -(-max(sc.final_lens) // spec.block_size)
    return _table([a.table(r) for r in sc.seqs], width), sc.final_lens


def test_prefix_workload_is_one_group_sharing_the_prompt():
    # 50 requests behind one 800-token system prompt (50 full blocks at B = 16);
    # the last request is a fork of request 0 and shares more with it, but not
    # with the others, so the group's prefix is the 50 prompt blocks.
    s = W.spec("prefix_13b")
    tables, lens = _prefix_layout(s)
    gs, mem, pb = prefix_groups(tables, lens, s.block_size)
    assert gs == [0, 50] and mem == list(range(50))
    assert pb == [800 // 16] * 50


def _lcp_full(ta, tb, la, lb, B):
    n = 0
    while n < len(ta) and (n + 1) * B <= min(la, lb) and ta[n] == tb[n] and ta[n] >= 0:
        n += 1
    return n


@pytest.mark.parametrize("seed", range(6))
def test_pairwise_definition_on_random_fork_trees(seed):
    # Layouts from random allocate / fork / append runs; the group prefix must
    # equal the smallest pairwise full-block common prefix of its members, and
    # no row left out may share a full first block with min_members - 1 others.
    rng = np.random.default_rng(seed)
    B = 4
    a = BlockAllocator(400, B)
    seqs = []
    for i in range(4):
        a.allocate(i, int(rng.integers(1, 20)))
        seqs.append(i)
    nxt = 4
    for _ in range(30):
        op = rng.integers(3)
        if op == 0:
            src = int(rng.choice(seqs))
            a.fork(src, nxt)
            seqs.append(nxt)
            nxt += 1
        else:
            r = int(rng.choice(seqs))
            for _ in range(int(rng.integers(1, 6))):
                a.append_slot(r)
    rows = [a.table(r) for r in seqs]
    lens = [a.num_tokens[r] for r in seqs]
    width = max(len(r) for r in rows)
    tables = _table(rows, width)
    for mm in (2, 3):
        gs, mem, pb = prefix_groups(tables, lens, B, min_members=mm)
        grouped = set(mem)
        for g in range(len(gs) - 1):
            m = mem[gs[g]:gs[g + 1]]
            assert len(m) >= mm and m == sorted(m)
            want = min(_lcp_full(rows[x], rows[y], lens[x], lens[y], B)
                       for x, y in itertools.combinations(m, 2))
            assert all(pb[x] == want for x in m) and want >= 1
        for x in range(len(seqs)):
            if x in grouped:
                continue
            assert pb[x] == 0
            if lens[x] >= B:
                same = [y for y in range(len(seqs)) if lens[y] >= B and rows[y][0] == rows[x][0]]
                assert len(same) < mm
