"""Pins of the prefix cache (oracle/radix.py) and the utilisation figures.

"RadixAttention — reuse a shared prefix" and "Managing the KV cache" (the
third page); "Shared System Prompts & Prefix Caching" (PagedAttention and KV
Cache Management).
"""
import random

import pytest

from oracle.allocator import ERR_EXISTS, ERR_INVALID, AllocError, BlockAllocator
from oracle.radix import PrefixCache, allocate_prefix


def test_hand_worked_cache_life():
    # B = 2, 16 blocks, FIFO from 0.
    a = BlockAllocator(16, 2)
    c = PrefixCache(a)
    a.allocate(1, 6)                                   # blocks 0, 1, 2
    assert c.insert(1, [1, 2, 3, 4, 5, 6]) == 3        # three full blocks cached
    assert a.refcount[:3] == [2, 2, 2]
    assert c.match([1, 2, 3, 4, 9, 9]) == [0, 1]       # the run stops at (9, 9)
    assert allocate_prefix(a, 2, [0, 1], 5) == [0, 1, 3]  # suffix block is fresh
    assert a.refcount[:4] == [3, 3, 2, 1]
    a.free(1)
    assert a.refcount[:4] == [2, 2, 1, 1]
    assert c.evict(5) == [2]                           # only (5, 6) is held by the cache alone
    assert c.nodes == 2
    a.free(2)
    assert c.evict(5) == [1, 0]                        # leaf first, then its parent
    assert c.nodes == 0 and a.num_free() == 16


def test_lru_order_and_ties():
    a = BlockAllocator(8, 1)
    c = PrefixCache(a)
    a.allocate(1, 1)
    a.allocate(2, 1)
    c.insert(1, [7])                                   # clock 1: node (7) on block 0
    c.insert(2, [8])                                   # clock 2: node (8) on block 1
    a.free(1)
    a.free(2)
    c.match([7])                                       # clock 3: (7) used again
    assert c.evict(1) == [1]                           # (8) is the least recently used
    a.allocate(3, 1)
    a.allocate(4, 1)
    c.insert(3, [5])                                   # clock 4: (5) on block 2
    c.match([7])                                       # clock 5: (7) used
    c.insert(4, [6])                                   # clock 6: (6) on block 3
    a.free(3)
    a.free(4)
    assert c.evict(3) == [2, 0, 3]                     # last use 4, 5, 6


def test_allocate_prefix_errors_change_nothing():
    a = BlockAllocator(4, 2)
    a.allocate(1, 4)
    before = (list(a.refcount), list(a.free_list))
    for args, code in [((1, [0], 2), ERR_EXISTS), ((2, [0, 1], 3), ERR_INVALID), ((2, [3], 2), ERR_INVALID)]:
        with pytest.raises(AllocError) as e:
            allocate_prefix(a, *args)
        assert e.value.code == code
        assert (list(a.refcount), list(a.free_list)) == before


@pytest.mark.parametrize("seed", range(5))
def test_match_is_longest_cached_prefix_by_brute_force(seed):
    # With nothing evicted, match(t) is the longest common full-block prefix of
    # t with any inserted sequence, and it returns the first inserter's blocks.
    rng = random.Random(seed)
    B = rng.choice([1, 2, 4])
    a = BlockAllocator(4000, B)
    c = PrefixCache(a)
    inserted = []  # (tokens, blocks of the sequence that first cached them)
    base = [rng.randint(0, 3) for _ in range(40)]
    for i in range(25):
        cut = rng.randint(0, 40)
        toks = base[:cut] + [rng.randint(0, 3) for _ in range(rng.randint(0, 20))]
        a.allocate(i, len(toks))
        c.insert(i, toks)
        inserted.append((toks, a.table(i)))
    for _ in range(60):
        cut = rng.randint(0, 40)
        q = base[:cut] + [rng.randint(0, 3) for _ in range(rng.randint(0, 12))]
        got = c.match(q)
        best = 0
        for toks, _ in inserted:
            n = 0
            while (n + 1) * B <= min(len(q), len(toks)) and q[n * B:(n + 1) * B] == toks[n * B:(n + 1) * B]:
                n += 1
            best = max(best, n)
        assert len(got) == best
        # block j belongs to the first inserted sequence sharing q's first j + 1 blocks
        for j, blk in enumerate(got):
            first = next(tb for toks, tb in inserted if toks[:(j + 1) * B] == q[:(j + 1) * B])
            assert blk == first[j]


def test_utilisation_figures_of_a_shared_prompt():
    # 5 requests behind a 4-block prompt (B = 4), each with a private 6-token
    # suffix: without sharing each holds 4 + 2 blocks (30); with sharing the
    # prompt is stored once: 4 + 5 * 2 = 14 blocks, saving 1 - 14/30.
    a = BlockAllocator(64, 4)
    a.allocate(100, 16)
    for r in range(5):
        a.fork(100, r)
        for _ in range(6):
            a.append_slot(r)
    a.free(100)
    st = a.stats()
    assert st["used"] == 14 and st["table_blocks"] == 30 and st["sequences"] == 5
    assert st["saved"] == pytest.approx(1 - 14 / 30)
    assert st["tokens"] == 16 + 5 * 6
    waste = st["used"] * 4 - st["tokens"]
    assert waste == 5 * 2 and waste <= 3 * st["sequences"]
