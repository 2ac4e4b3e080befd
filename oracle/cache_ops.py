"""Cache writes and block copies, on raw storage. Test infrastructure only.

reshape_and_cache: during generation each new token's K and V go into the
sequence's current (last) block ("How Block Paging Operates During
Generation", "PagedAttention and KV Cache Management"). A token's slot is a
flat index into the pool: slot = physical_block * B + offset, so its K/V row
lives at pool[slot // B, h, slot % B, :]. A negative slot marks a padding
token and is skipped. The fp8 variant stores the e4m3 code of x / scale[h],
the quotient formed in fp32 (an fp8 cache halves the bytes per element:
"Planning capacity when context gets long", "KV-Cache Management and
PagedAttention").

copy_blocks: the device half of copy-on-write. When a branch writes into a
shared block, the engine takes a fresh block and copies the shared block's B
token slots into it ("Parallel Sampling & Beam Search via Copy-on-Write",
"PagedAttention and KV Cache Management"). With one pool per layer that is
every slot of the block, K and V, all heads, bit for bit. All copies of one
call read the pool as it was before the call.
"""
from __future__ import annotations

import numpy as np

from .numerics import encode_e4m3, to_float32


def reshape_and_cache(k, v, k_pool, v_pool, slot_mapping, block_size: int):
    """New (k_pool, v_pool) with token t's rows stored at slot_mapping[t].

    Raw arrays: k, v [T, Hk, D]; pools [NB, Hk, B, D], same element type.
    """
    k_pool = np.array(k_pool, copy=True)
    v_pool = np.array(v_pool, copy=True)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        k_pool[blk, :, off, :] = k[t]
        v_pool[blk, :, off, :] = v[t]
    return k_pool, v_pool


def reshape_and_cache_fp8(k, v, k_pool, v_pool, slot_mapping, block_size: int, kind: str,
                          k_scale, v_scale):
    """fp8 variant: pools hold uint8 e4m3 codes, k / v are raw f16 / bf16."""
    k_pool = np.array(k_pool, copy=True)
    v_pool = np.array(v_pool, copy=True)
    ks = np.asarray(k_scale, dtype=np.float32)
    vs = np.asarray(v_scale, dtype=np.float32)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        kq = to_float32(k[t], kind) / ks[:, None]  # fp32 quotient, per kv head
        vq = to_float32(v[t], kind) / vs[:, None]
        k_pool[blk, :, off, :] = encode_e4m3(kq)
        v_pool[blk, :, off, :] = encode_e4m3(vq)
    return k_pool, v_pool


def copy_blocks(k_pool, v_pool, pairs):
    """New (k_pool, v_pool) with block dst := block src for each (src, dst)."""
    k_old, v_old = np.asarray(k_pool), np.asarray(v_pool)
    k_new, v_new = k_old.copy(), v_old.copy()
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        k_new[dst] = k_old[src]
        v_new[dst] = v_old[src]
    return k_new, v_new


def slot_of(table_row, position: int, block_size: int) -> int:
    """Flat slot of a token position through a block table row."""
    return int(table_row[position // block_size]) * block_size + position % block_size
