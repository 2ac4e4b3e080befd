"""Prefix cache over a block allocator (radix tree of full blocks). Test
infrastructure only.

"RadixAttention — reuse a shared prefix" (the third page): cached prefixes
live in a radix tree, a shared beginning is a single branch, a new request
that matches a cached prefix reuses its blocks and only its own suffix takes
new memory. "Shared System Prompts & Prefix Caching" (PagedAttention and KV
Cache Management): the shared blocks are mapped into every matching
request's block table and reference-counted.

Structure (the plain reading, at block granularity, since a block is the unit
that can be shared):
  * A node is one full block: its B token ids and its physical block. The
    root is empty; a node's children are keyed by the next block's tokens.
  * insert(seq, tokens): walk the sequence's full blocks from the root; a
    block whose tokens already have a node is left alone (the cached block is
    kept); otherwise a node is added for the sequence's block and the cache
    takes one reference on it. Returns the number of nodes added.
  * match(tokens): the blocks of the longest run of leading full blocks found
    in the tree; every node on the run is touched (last use := the clock).
  * evict(n): up to n times, release the least recently used leaf whose block
    no one but the cache references (ties: the older node first); its block
    returns to the free list and its parent may become a leaf.
  * The clock advances by one per insert and per match call.

allocate_prefix(seq, blocks, tokens) on the allocator side creates a sequence
whose first len(blocks) table entries are the given blocks (one more
reference each) and whose remaining ceil(tokens / B) - len(blocks) blocks are
fresh.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

from .allocator import ERR_EXISTS, ERR_INVALID, ERR_OOM, AllocError, BlockAllocator


class _Node:
    __slots__ = ("key", "block", "parent", "children", "last", "born")

    def __init__(self, key, block, parent, born):
        self.key = key
        self.block = block
        self.parent = parent
        self.children: Dict[Tuple[int, ...], "_Node"] = {}
        self.last = born
        self.born = born


def allocate_prefix(a: BlockAllocator, seq: int, blocks: Sequence[int], num_tokens: int) -> List[int]:
    """A new sequence starting with the cached `blocks`, the rest fresh."""
    if seq in a.tables or seq in a.swapped:
        raise AllocError(ERR_EXISTS, f"sequence {seq} exists")
    n = -(-num_tokens // a.block_size)
    if num_tokens < 0 or len(blocks) * a.block_size > num_tokens:
        raise AllocError(ERR_INVALID, "cached blocks exceed the token count")
    if any(b < 0 or b >= a.num_blocks or a.refcount[b] <= 0 for b in blocks):
        raise AllocError(ERR_INVALID, "cached block not in use")
    a._need(n - len(blocks))
    for b in blocks:
        a.refcount[b] += 1
    a.tables[seq] = list(blocks) + [a._take() for _ in range(n - len(blocks))]
    a.num_tokens[seq] = num_tokens
    return list(a.tables[seq])


class PrefixCache:
    def __init__(self, alloc: BlockAllocator):
        self.a = alloc
        self.B = alloc.block_size
        self.clock = 0
        self.born = 0
        self.root = _Node((), -1, None, 0)
        self.nodes = 0

    def _chunks(self, tokens: Sequence[int]):
        B = self.B
        return [tuple(int(x) for x in tokens[i * B:(i + 1) * B]) for i in range(len(tokens) // B)]

    def insert(self, seq: int, tokens: Sequence[int]) -> int:
        table = self.a.table(seq)
        if len(tokens) > self.a.num_tokens[seq]:
            raise AllocError(ERR_INVALID, "more tokens than the sequence holds")
        self.clock += 1
        node, added = self.root, 0
        for i, key in enumerate(self._chunks(tokens)):
            child = node.children.get(key)
            if child is None:
                self.born += 1
                child = _Node(key, table[i], node, self.born)
                child.last = self.clock
                node.children[key] = child
                self.a.refcount[table[i]] += 1
                self.nodes += 1
                added += 1
            else:
                child.last = self.clock
            node = child
        return added

    def match(self, tokens: Sequence[int]) -> List[int]:
        self.clock += 1
        node, out = self.root, []
        for key in self._chunks(tokens):
            child = node.children.get(key)
            if child is None:
                break
            child.last = self.clock
            out.append(child.block)
            node = child
        return out

    def _leaves(self):
        stack, out = list(self.root.children.values()), []
        while stack:
            n = stack.pop()
            if n.children:
                stack.extend(n.children.values())
            else:
                out.append(n)
        return out

    def evict(self, n: int) -> List[int]:
        freed = []
        while len(freed) < n:
            cands = [x for x in self._leaves() if self.a.refcount[x.block] == 1]
            if not cands:
                break
            victim = min(cands, key=lambda x: (x.last, x.born))
            del victim.parent.children[victim.key]
            self.nodes -= 1
            self.a._drop(victim.block)
            freed.append(victim.block)
        return freed
