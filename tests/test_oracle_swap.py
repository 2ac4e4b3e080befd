"""Pins of preemption by swapping (oracle/allocator.py swap_out / swap_in,
oracle/cache_ops.py swap_out / swap_in).

Preemption by swapping: "Preemption and eviction" (KV-Cache Management page,
"PagedAttention: treat the cache like virtual memory") and "Preemption & GPU
Swapping" ("PagedAttention and KV Cache Management").
"""
import numpy as np
import pytest

from oracle import cache_ops
from oracle.allocator import (ERR_EXISTS, ERR_OOM, ERR_UNKNOWN_SEQ, AllocError, BlockAllocator)


def test_hand_worked_swap_sequence():
    # B = 4, 10 blocks, FIFO free list 0..9.
    a = BlockAllocator(10, 4)
    assert a.allocate(1, 6) == [0, 1]
    assert a.allocate(2, 3) == [2]
    a.fork(1, 3)                        # blocks 0, 1 now have two references
    assert a.swap_out(1) == [0, 1]      # one reference each goes: nothing is freed
    assert a.refcount[:3] == [1, 1, 1] and a.num_free() == 7
    assert a.swap_out(3) == [0, 1]      # last references: 0 and 1 go to the tail
    assert list(a.free_list) == [3, 4, 5, 6, 7, 8, 9, 0, 1]
    assert a.swap_in(1) == [3, 4]       # fresh blocks from the head, in table order
    assert a.num_tokens[1] == 6 and a.table(1) == [3, 4]
    assert a.swap_in(3) == [5, 6]
    a.append_slot(3)                    # 7th token: block 6 has room
    assert a.table(3) == [5, 6] and a.num_tokens[3] == 7


def test_swapped_sequence_is_unknown_but_its_id_is_taken():
    a = BlockAllocator(4, 4)
    a.allocate(7, 5)
    a.swap_out(7)
    for call in (lambda: a.append_slot(7), lambda: a.fork(7, 8), lambda: a.swap_out(7), lambda: a.table(7)):
        with pytest.raises(AllocError) as e:
            call()
        assert e.value.code == ERR_UNKNOWN_SEQ
    with pytest.raises(AllocError) as e:
        a.allocate(7, 1)
    assert e.value.code == ERR_EXISTS
    with pytest.raises(AllocError) as e:
        a.swap_in(9)
    assert e.value.code == ERR_UNKNOWN_SEQ
    a.free(7)                           # forgets it
    a.allocate(7, 1)


def test_swap_in_out_of_blocks_changes_nothing():
    a = BlockAllocator(3, 4)
    a.allocate(1, 12)                   # all three blocks
    a.swap_out(1)
    a.allocate(2, 5)                    # two of them
    before = (list(a.free_list), list(a.refcount), dict(a.swapped))
    with pytest.raises(AllocError) as e:
        a.swap_in(1)
    assert e.value.code == ERR_OOM
    assert (list(a.free_list), list(a.refcount), dict(a.swapped)) == before


def test_record_layout_by_hand():
    # pool [NB=3, Hk=2, B=2, D=2] of uint16 with value = flat index; record of
    # block 2 = its 8 K values (row-major) then its 8 V values, as bytes.
    k = np.arange(24, dtype=np.uint16).reshape(3, 2, 2, 2)
    v = (1000 + np.arange(24, dtype=np.uint16)).reshape(3, 2, 2, 2)
    rec = cache_ops.swap_out(k, v, [2])
    assert rec.shape == (1, 32)
    assert rec[0].view(np.uint16).tolist() == list(range(16, 24)) + list(range(1016, 1024))


@pytest.mark.parametrize("dtype", [np.uint16, np.uint8])
def test_round_trip_into_other_blocks(dtype):
    rng = np.random.default_rng(3)
    k = rng.integers(0, np.iinfo(dtype).max, size=(9, 3, 4, 8), dtype=dtype)
    v = rng.integers(0, np.iinfo(dtype).max, size=(9, 3, 4, 8), dtype=dtype)
    src, dst = [4, 0, 7], [1, 8, 2]
    rec = cache_ops.swap_out(k, v, src)
    k2, v2 = cache_ops.swap_in(rec, k, v, dst)
    for s, d in zip(src, dst):
        assert np.array_equal(k2[d], k[s]) and np.array_equal(v2[d], v[s])
    untouched = [b for b in range(9) if b not in dst]
    assert np.array_equal(k2[untouched], k[untouched]) and np.array_equal(v2[untouched], v[untouched])
