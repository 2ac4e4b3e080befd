"""KV-cache byte counts. Test infrastructure only.

"Why the cache exists, and why it's so hungry" ("KV-Cache Management and
PagedAttention") and "The KV Cache Size Equation" ("PagedAttention and KV
Cache Management") give the size of the cache as the product of: 2 (one K and
one V row), the number of layers, the number of KV heads, the head dimension,
the number of tokens, the bytes per element and the batch size. The 13B
example writes the head term as the hidden size, which is the same number
only when every query head has its own KV head; the formula here always uses
num_kv_heads * head_dim.

A physical block holds B tokens' K and V rows ("How Block Paging Operates
During Generation"); with one pool per layer a block of one layer's pool is
2 * B * num_kv_heads * head_dim * dtype_bytes bytes.
"""
from __future__ import annotations


def kv_bytes(num_layers: int, num_kv_heads: int, head_dim: int, seq_len: int,
             dtype_bytes: int, batch: int = 1) -> int:
    return 2 * num_layers * num_kv_heads * head_dim * seq_len * dtype_bytes * batch


def blocks_for(num_tokens: int, block_size: int) -> int:
    return -(-num_tokens // block_size)


def block_bytes(block_size: int, num_kv_heads: int, head_dim: int, dtype_bytes: int,
                num_layers: int = 1) -> int:
    return 2 * block_size * num_layers * num_kv_heads * head_dim * dtype_bytes


def decode_kv_bytes(context_lens, num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    """K and V bytes one decode step over one layer must read: every stored
    token of every sequence, once."""
    return sum(kv_bytes(1, num_kv_heads, head_dim, int(L), dtype_bytes) for L in context_lens)
