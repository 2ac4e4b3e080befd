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

swap_out / swap_in: the device half of preemption by swapping ("Preemption
and eviction", KV-Cache Management page; "Preemption & GPU Swapping",
"PagedAttention and KV Cache Management"): a preempted sequence's blocks go to
host memory and later come back, possibly into other blocks. Host layout:
one record per block in the order given, the block's K bytes ([Hk, B, D],
row-major) then its V bytes.
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


def swap_out(k_pool, v_pool, blocks) -> np.ndarray:
    """uint8 [n, 2 * Hk * B * D * e]: the records of the given blocks."""
    recs = []
    for blk in blocks:
        kb = np.ascontiguousarray(k_pool[int(blk)]).view(np.uint8).reshape(-1)
        vb = np.ascontiguousarray(v_pool[int(blk)]).view(np.uint8).reshape(-1)
        recs.append(np.concatenate([kb, vb]))
    width = 2 * int(np.prod(k_pool.shape[1:])) * k_pool.dtype.itemsize
    return np.stack(recs) if recs else np.zeros((0, width), dtype=np.uint8)


def swap_in(records, k_pool, v_pool, blocks):
    """New (k_pool, v_pool) with record i written into block blocks[i]."""
    k_pool = np.array(k_pool, copy=True)
    v_pool = np.array(v_pool, copy=True)
    half = records.shape[1] // 2 if len(blocks) else 0
    for i, blk in enumerate(blocks):
        k_pool[int(blk)] = records[i, :half].view(k_pool.dtype).reshape(k_pool.shape[1:])
        v_pool[int(blk)] = records[i, half:].view(v_pool.dtype).reshape(v_pool.shape[1:])
    return k_pool, v_pool


def slot_of(table_row, position: int, block_size: int) -> int:
    """Flat slot of a token position through a block table row."""
    return int(table_row[position // block_size]) * block_size + position % block_size
