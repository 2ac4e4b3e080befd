"""Block allocator semantics. Test infrastructure only.

Follows "Hands-On Implementation: Building a PagedAttention Block Allocator in
Python" and "How Block Paging Operates During Generation" of "PagedAttention
and KV Cache Management", in a structure of its own:

  * The pool has N blocks of B token slots. Free blocks sit in a list; a new
    block is taken from the HEAD of that list and a released block goes to its
    TAIL (first in, first out), and a taken block starts with reference count
    1. The printed demo run of that section fixes this order: after one
    request takes blocks 0 and 1, a copy-on-write takes block 2.
  * A sequence of n prompt tokens takes ceil(n / B) blocks, in table order
    (on-demand allocation: a 25-token prompt at B = 16 takes 2 blocks).
  * Appending a token writes into the last block while it has room; at a
    block boundary a new block is taken (boundary allocation).
  * Forking copies the table and adds one reference to each block; it takes no
    block (zero-copy parallel sampling).
  * When a sequence must write into a block that another sequence also
    references, it first takes a fresh block, the B slots are copied into it
    (the device does this: the returned (src, dst) pair), the shared block
    loses one reference and the table points at the copy (copy-on-write).
  * Freeing a sequence drops one reference on each block in table order; a
    block whose count reaches 0 returns to the free list.

Preemption by swapping ("Preemption and eviction" of "PagedAttention: treat
the cache like virtual memory" on the KV-Cache Management page; "Preemption &
GPU Swapping" of "PagedAttention and KV Cache Management"): a swapped-out
sequence gives up its blocks (its data goes to host memory first) and keeps
only its token count; swapping it in takes fresh blocks, in table order,
which the device fills from host memory.

Readings where the listing is silent or would misbehave (each is a status
code here, never a partial update):
  * Copy-on-write happens only when the slot to be written lies in a shared
    block, i.e. the last block is shared AND has room. A shared full last
    block stays shared and the token goes to a new block, since nothing in
    the shared block changes (the copy-on-write paragraph triggers the copy
    when a branch would change a shared block). The demo run is unchanged.
  * Appending to a sequence with no blocks takes a new block.
  * Running out of blocks raises AllocError(OOM) and changes nothing (the
    listing raises MemoryError, possibly after taking some blocks).
  * Freeing an unknown sequence is a no-op (as in the listing); other calls
    on an unknown sequence raise UNKNOWN_SEQ; creating an existing one
    raises EXISTS; a reference count that would go below 0 raises DOUBLE_FREE.
  * Swap: swapping out drops one reference on each block (in table order,
    shared blocks included: the host copy is the sequence's own) and returns
    the blocks to copy; a swapped-out sequence is unknown to every other call
    but free (which forgets it) and swap_in, and its id stays taken. Swapping
    in needs ceil(tokens / B) free blocks (OOM otherwise, nothing changes).
"""
from __future__ import annotations

import collections
from typing import Dict, List, Optional, Sequence, Tuple

OK, ERR_INVALID, ERR_OOM, ERR_UNKNOWN_SEQ, ERR_EXISTS, ERR_DOUBLE_FREE = 0, -1, -3, -4, -5, -6


class AllocError(Exception):
    def __init__(self, code: int, what: str):
        super().__init__(what)
        self.code = code


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocError(ERR_INVALID, "num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise AllocError(ERR_INVALID, "free_order must be a permutation of the block ids")
        self.block_size = block_size
        self.num_blocks = num_blocks
        self.free_list = collections.deque(order)
        self.refcount = [0] * num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.num_tokens: Dict[int, int] = {}
        self.swapped: Dict[int, int] = {}  # swapped-out sequence -> tokens

    # -- block level ---------------------------------------------------------
    def _take(self) -> int:
        blk = self.free_list.popleft()
        self.refcount[blk] = 1
        return blk

    def _drop(self, blk: int) -> None:
        if self.refcount[blk] <= 0:
            raise AllocError(ERR_DOUBLE_FREE, f"block {blk} has no reference left")
        self.refcount[blk] -= 1
        if self.refcount[blk] == 0:
            self.free_list.append(blk)

    def _need(self, n: int) -> None:
        if n > len(self.free_list):
            raise AllocError(ERR_OOM, f"need {n} free blocks, have {len(self.free_list)}")

    def _table(self, seq: int) -> List[int]:
        if seq not in self.tables:
            raise AllocError(ERR_UNKNOWN_SEQ, f"unknown sequence {seq}")
        return self.tables[seq]

    # -- sequence level ------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> List[int]:
        if seq in self.tables or seq in self.swapped:
            raise AllocError(ERR_EXISTS, f"sequence {seq} exists")
        if num_tokens < 0:
            raise AllocError(ERR_INVALID, "negative token count")
        n = -(-num_tokens // self.block_size)
        self._need(n)
        self.tables[seq] = [self._take() for _ in range(n)]
        self.num_tokens[seq] = num_tokens
        return list(self.tables[seq])

    def append_slot(self, seq: int) -> Tuple[int, int, int]:
        """(slot, cow_src, cow_dst) for one new token; cow_* = -1 without a copy."""
        table = self._table(seq)
        B = self.block_size
        held = self.num_tokens[seq]
        room = len(table) * B - held  # free slots left in the last block
        cow = (-1, -1)
        if room == 0:
            self._need(1)
            blk = self._take()
            table.append(blk)
            offset = 0
        else:
            blk = table[-1]
            offset = B - room
            if self.refcount[blk] > 1:
                self._need(1)
                fresh = self._take()
                self.refcount[blk] -= 1
                table[-1] = fresh
                cow = (blk, fresh)
                blk = fresh
        self.num_tokens[seq] = held + 1
        return blk * B + offset, cow[0], cow[1]

    def append_tokens(self, seq: int, count: int) -> List[Tuple[int, int, int]]:
        return [self.append_slot(seq) for _ in range(count)]

    def fork(self, src: int, dst: int) -> None:
        table = self._table(src)
        if dst in self.tables or dst in self.swapped:
            raise AllocError(ERR_EXISTS, f"sequence {dst} exists")
        for blk in table:
            self.refcount[blk] += 1
        self.tables[dst] = list(table)
        self.num_tokens[dst] = self.num_tokens[src]

    def free(self, seq: int) -> None:
        self.swapped.pop(seq, None)
        if seq not in self.tables:
            return
        for blk in self.tables[seq]:
            self._drop(blk)
        del self.tables[seq]
        del self.num_tokens[seq]

    def swap_out(self, seq: int) -> List[int]:
        """The sequence's blocks in table order (to copy to host memory before
        they are reused); each loses this sequence's reference."""
        table = self._table(seq)
        for blk in table:
            self._drop(blk)
        self.swapped[seq] = self.num_tokens.pop(seq)
        del self.tables[seq]
        return list(table)

    def swap_in(self, seq: int) -> List[int]:
        """Fresh blocks for a swapped-out sequence, in table order (to fill
        from host memory)."""
        if seq not in self.swapped:
            raise AllocError(ERR_UNKNOWN_SEQ, f"sequence {seq} is not swapped out")
        n_tok = self.swapped[seq]
        n = -(-n_tok // self.block_size)
        self._need(n)
        del self.swapped[seq]
        self.tables[seq] = [self._take() for _ in range(n)]
        self.num_tokens[seq] = n_tok
        return list(self.tables[seq])

    # -- queries -------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_list)

    def table(self, seq: int) -> List[int]:
        return list(self._table(seq))

    def stats(self) -> Dict[str, float]:
        """Free / used / shared block counts and slot utilisation.

        Utilisation is tokens held in used blocks over their slots, each
        physical block counted once (the packing figure of the widget in
        "Managing the KV cache" divides held tokens by reserved blocks).
        """
        B = self.block_size
        fill = {}
        for seq, table in self.tables.items():
            n = self.num_tokens[seq]
            for i, blk in enumerate(table):
                fill[blk] = max(fill.get(blk, 0), max(0, min(B, n - i * B)))
        used = sum(1 for r in self.refcount if r > 0)
        shared = sum(1 for r in self.refcount if r > 1)
        tokens = sum(fill.values())
        table_blocks = sum(len(t) for t in self.tables.values())
        return {"free": self.num_free(), "used": used, "shared": shared, "tokens": tokens,
                "utilisation": (tokens / (used * B)) if used else 1.0,
                "table_blocks": table_blocks, "sequences": len(self.tables),
                "saved": (1.0 - used / table_blocks) if table_blocks else 0.0}

    def run(self, ops) -> None:
        """Execute ("allocate", seq, n) / ("fork", src, dst) / ("free", seq) /
        ("append", seq, count) operations in order."""
        for op in ops:
            if op[0] == "allocate":
                self.allocate(op[1], op[2])
            elif op[0] == "fork":
                self.fork(op[1], op[2])
            elif op[0] == "free":
                self.free(op[1])
            elif op[0] == "append":
                self.append_tokens(op[1], op[2])
            elif op[0] == "swap_out":
                self.swap_out(op[1])
            elif op[0] == "swap_in":
                self.swap_in(op[1])
            else:
                raise ValueError(op)
