"""Decode-step attention over a paged KV cache, in fp64. Test infrastructure only.

What it computes ("PagedAttention: treat the cache like virtual memory",
"KV-Cache Management and PagedAttention"; "Under the Hood: The PagedAttention
CUDA Kernel", "PagedAttention and KV Cache Management"): the cache of a
sequence is split into fixed-size blocks of B tokens; a per-sequence block
table maps logical block i (tokens iB .. iB+B-1) to a physical block of the
pool; attention for the newest query gathers K and V through that table. The
paging changes only where bytes live, so the result is plain single-query
softmax attention over the sequence's reassembled K and V:

    K_s[t] = k_pool[table[s][t // B], h, t % B, :],  same for V
    x_t    = scale * <q[s, i], K_s[t]>
    out[s, i] = sum_t exp(x_t - max x) V_s[t] / sum_t exp(x_t - max x)

with kv head h = i // g for query head i and g = Hq / Hk query heads per
kv head (grouped-query attention, "The KV Cache Size Equation": n_kv_heads is
much smaller than n_q_heads). A sequence of length 0 attends to nothing and
its output is 0. Slots past the sequence length (the unused tail of the last
block; the block-table diagram's third block uses 9 of its 16 slots) are
never read.
"""
from __future__ import annotations

from typing import Iterable, Optional

import numpy as np

from .numerics import widen


def gather_sequence(pool, table_row, length: int, block_size: int, kv_head: int,
                    kind: str, scale_h: Optional[float] = None) -> np.ndarray:
    """Reassemble one sequence's contiguous [L, D] fp64 rows for one kv head."""
    t = np.arange(length, dtype=np.int64)
    blocks = np.asarray(table_row, dtype=np.int64)[t // block_size]
    rows = np.asarray(pool)[blocks, kv_head, t % block_size, :]
    vals = widen(rows, kind)
    if scale_h is not None:
        vals = vals * float(scale_h)
    return vals.reshape(length, -1)


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale: float, block_size: int,
                 q_kind: str, cache_kind: str, k_scale=None, v_scale=None,
                 seqs: Optional[Iterable[int]] = None) -> np.ndarray:
    """fp64 output [S, Hq, D] (rows of sequences not in `seqs` stay 0).

    q: raw [S, Hq, D] (float16 array or bf16 bits); pools: raw [NB, Hk, B, D];
    block_tables int [S, W]; context_lens int [S]; for fp8 caches, k_scale /
    v_scale are the per-kv-head dequantisation scales (value = decode(code)
    * scale).
    """
    q = np.asarray(q)
    S, Hq, D = q.shape
    Hk = np.asarray(k_pool).shape[1]
    assert Hq % Hk == 0
    g = Hq // Hk
    out = np.zeros((S, Hq, D), dtype=np.float64)
    seqs = range(S) if seqs is None else seqs
    for s in seqs:
        L = int(context_lens[s])
        if L == 0:
            continue
        for h in range(Hk):
            ks = None if k_scale is None else float(np.asarray(k_scale)[h])
            vs = None if v_scale is None else float(np.asarray(v_scale)[h])
            K = gather_sequence(k_pool, block_tables[s], L, block_size, h, cache_kind, ks)
            V = gather_sequence(v_pool, block_tables[s], L, block_size, h, cache_kind, vs)
            for i in range(h * g, (h + 1) * g):
                qi = widen(q[s, i], q_kind)
                x = scale * (K @ qi)
                w = np.exp(x - x.max())
                out[s, i] = (w @ V) / w.sum()
    return out


def contiguous_attention_loops(qv, K, V, scale: float):
    """Single-query softmax attention over plain Python lists, for tiny cases.

    An independent routine (no numpy, no paging) used to pin paged_decode:
    dot products by explicit loops, softmax with math.exp and math.fsum.
    """
    import math

    L = len(K)
    if L == 0:
        return [0.0] * len(qv)
    x = [scale * math.fsum(a * b for a, b in zip(qv, K[t])) for t in range(L)]
    m = max(x)
    w = [math.exp(v - m) for v in x]
    l = math.fsum(w)
    D = len(V[0])
    return [math.fsum(w[t] * V[t][d] for t in range(L)) / l for d in range(D)]


def paged_prefill(q, k_pool, v_pool, block_tables, context_lens, q_start, scale: float, block_size: int,
                  q_kind: str, cache_kind: str, k_scale=None, v_scale=None,
                  seqs: Optional[Iterable[int]] = None) -> np.ndarray:
    """Causal attention of several new query tokens per sequence, fp64 [T, Hq, D].

    Several new tokens of a sequence attend over its paged cache in one call
    when a prompt (or a chunk of it) is processed after its K/V were written
    to the blocks allocated for it ("How Block Paging Operates During
    Generation": a request's prompt gets its blocks when it starts; "Dynamic
    Request Insertion": a waiting request's prefill joins the running
    iteration), or when speculative tokens are verified (the takeaways name
    speculative decoding among the uses of shared blocks). Plain reading:
    sequence s has n_s = q_start[s + 1] - q_start[s] new tokens, the last
    n_s of its L_s = context_lens[s] tokens; query row q_start[s] + j holds
    the token at position p = L_s - n_s + j, which attends (causally) to the
    positions 0 .. p of the same sequence, through the block table exactly
    as the decode query does. n_s = 1 is the decode step.
    """
    q = np.asarray(q)
    T, Hq, D = q.shape
    Hk = np.asarray(k_pool).shape[1]
    g = Hq // Hk
    out = np.zeros((T, Hq, D), dtype=np.float64)
    q_start = np.asarray(q_start, dtype=np.int64)
    S = len(q_start) - 1
    seqs = range(S) if seqs is None else seqs
    for s in seqs:
        L = int(context_lens[s])
        n = int(q_start[s + 1] - q_start[s])
        assert 0 <= n <= L
        if n == 0:
            continue
        for h in range(Hk):
            ks = None if k_scale is None else float(np.asarray(k_scale)[h])
            vs = None if v_scale is None else float(np.asarray(v_scale)[h])
            K = gather_sequence(k_pool, block_tables[s], L, block_size, h, cache_kind, ks)
            V = gather_sequence(v_pool, block_tables[s], L, block_size, h, cache_kind, vs)
            for j in range(n):
                p = L - n + j
                for i in range(h * g, (h + 1) * g):
                    qi = widen(q[q_start[s] + j, i], q_kind)
                    x = scale * (K[:p + 1] @ qi)
                    w = np.exp(x - x.max())
                    out[q_start[s] + j, i] = (w @ V[:p + 1]) / w.sum()
    return out
