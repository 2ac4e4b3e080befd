"""Pins for oracle.allocator: the pages' worked demo run and invariants."""
import os
import random

import pytest

from oracle.allocator import (BlockAllocator, AllocError, ERR_OOM, ERR_UNKNOWN_SEQ, ERR_EXISTS,
                              ERR_DOUBLE_FREE)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "allocator_demo.txt")


def read_golden():
    steps = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, *kv = line.split()
        steps[name] = {k: v for k, v in (x.split("=") for x in kv)}
    return steps


def _ids(s):
    return [int(x) for x in s.split(",")]


def run_demo(make, table, num_free, allocate, fork, append, free):
    """Drive an allocator through the demo run and compare with the golden file."""
    g = read_golden()
    n, B = int(g["pool"]["num_blocks"]), int(g["pool"]["block_size"])
    assert n * B == int(g["pool"]["capacity_tokens"])
    a = make(n, B)
    A, Bq = 1, 2
    allocate(a, A, 6)
    assert table(a, A) == _ids(g["allocate_A"]["table_A"])
    assert num_free(a) == int(g["allocate_A"]["free"])
    fork(a, A, Bq)
    assert table(a, Bq) == _ids(g["fork_B"]["table_B"])
    assert num_free(a) == int(g["fork_B"]["free"])
    append(a, A)
    assert table(a, A) == _ids(g["append_A"]["table_A"])
    assert table(a, Bq) == _ids(g["append_A"]["table_B"])
    assert num_free(a) == int(g["append_A"]["free"])
    free(a, A)
    free(a, Bq)
    assert num_free(a) == int(g["free_A_B"]["free"])


def test_demo_run_matches_pages():
    run_demo(lambda n, B: BlockAllocator(n, B), lambda a, s: a.table(s), lambda a: a.num_free(),
             lambda a, s, n: a.allocate(s, n), lambda a, s, d: a.fork(s, d),
             lambda a, s: a.append_slot(s), lambda a, s: a.free(s))


def test_demo_cow_pair_and_slot():
    a = BlockAllocator(10, 4)
    a.allocate(1, 6)
    a.fork(1, 2)
    slot, src, dst = a.append_slot(1)
    assert (src, dst) == (1, 2)          # shared partial block 1 copied into fresh block 2
    assert slot == 2 * 4 + 2             # 7th token at offset 2 of block 2
    assert a.refcount[1] == 1 and a.refcount[0] == 2 and a.refcount[2] == 1


def test_fifo_free_list_order():
    a = BlockAllocator(6, 2)
    a.allocate(1, 4)      # blocks 0, 1
    a.allocate(2, 2)      # block 2
    a.free(1)             # 0 then 1 go to the tail: free list 3, 4, 5, 0, 1
    a.allocate(3, 10)
    assert a.table(3) == [3, 4, 5, 0, 1]


def test_prompt_of_25_tokens_takes_2_blocks():
    # on-demand allocation example: 25 prompt tokens at B = 16 need two blocks
    a = BlockAllocator(8, 16)
    assert len(a.allocate(1, 25)) == 2


def test_boundary_allocation_and_full_shared_block_stays_shared():
    a = BlockAllocator(8, 4)
    a.allocate(1, 4)                      # one full block
    a.fork(1, 2)
    slot, src, dst = a.append_slot(1)     # last block full: new block, no copy
    assert (src, dst) == (-1, -1) and slot == 1 * 4 + 0
    assert a.table(1) == [0, 1] and a.table(2) == [0]
    assert a.refcount[0] == 2


def test_append_to_empty_sequence_and_errors():
    a = BlockAllocator(2, 4)
    a.allocate(1, 0)
    assert a.table(1) == []
    assert a.append_slot(1) == (0, -1, -1)
    with pytest.raises(AllocError) as e:
        a.allocate(1, 3)
    assert e.value.code == ERR_EXISTS
    with pytest.raises(AllocError) as e:
        a.append_slot(99)
    assert e.value.code == ERR_UNKNOWN_SEQ
    a.free(99)                            # unknown free: no-op
    with pytest.raises(AllocError) as e:
        a.allocate(2, 9)                  # needs 3 of 1 free
    assert e.value.code == ERR_OOM
    assert a.num_free() == 1 and 2 not in a.tables   # nothing changed
    b = BlockAllocator(2, 4)
    b.allocate(1, 3)
    b._drop(0)                            # the only reference is gone
    with pytest.raises(AllocError) as e:
        b._drop(0)
    assert e.value.code == ERR_DOUBLE_FREE


def test_oom_on_copy_leaves_state_unchanged():
    a = BlockAllocator(2, 4)
    a.allocate(1, 6)                      # both blocks
    a.fork(1, 2)
    before = (a.table(1), a.table(2), list(a.refcount), a.num_tokens[1])
    with pytest.raises(AllocError) as e:
        a.append_slot(1)                  # must copy block 1, none free
    assert e.value.code == ERR_OOM
    assert (a.table(1), a.table(2), list(a.refcount), a.num_tokens[1]) == before


def test_invariants_under_random_ops():
    rng = random.Random(5)
    N, B = 64, 4
    a = BlockAllocator(N, B, free_order=rng.sample(range(N), N))
    live = []
    nxt = 0
    for step in range(3000):
        op = rng.random()
        try:
            if op < 0.25 or not live:
                a.allocate(nxt, rng.randint(0, 12))
                live.append(nxt)
                nxt += 1
            elif op < 0.35:
                a.fork(rng.choice(live), nxt)
                live.append(nxt)
                nxt += 1
            elif op < 0.5:
                s = rng.choice(live)
                a.free(s)
                live.remove(s)
            else:
                a.append_slot(rng.choice(live))
        except AllocError as e:
            assert e.code == ERR_OOM
        # every reference is a table entry, and every block is free xor referenced
        assert sum(a.refcount) == sum(len(t) for t in a.tables.values())
        assert a.num_free() + sum(1 for r in a.refcount if r > 0) == N
        assert all((r == 0) == (b in a.free_list) for b, r in enumerate(a.refcount))
        for s, t in a.tables.items():
            n = a.num_tokens[s]
            assert len(t) == -(-n // B)           # no over-reservation
            assert len(t) * B - n <= B - 1        # waste below one block
    for s in list(live):
        a.free(s)
    assert a.num_free() == N


def test_stats_utilisation():
    a = BlockAllocator(10, 4)
    a.allocate(1, 6)
    a.fork(1, 2)
    st = a.stats()
    assert st == {"free": 8, "used": 2, "shared": 2, "tokens": 6, "utilisation": 6 / 8,
                  "table_blocks": 4, "sequences": 2, "saved": 0.5}
