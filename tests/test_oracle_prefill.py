"""Pins of the multi-token (causal) paged attention oracle, paged_prefill."""
import numpy as np
import pytest

from oracle.attention import contiguous_attention_loops, paged_decode, paged_prefill


def _case(seed, S=3, Hq=4, Hk=2, D=8, B=4, lens=(9, 4, 13), nq=(3, 4, 1)):
    rng = np.random.default_rng(seed)
    NB = sum(-(-L // B) for L in lens) + 3
    perm = rng.permutation(NB)
    W = max(-(-L // B) for L in lens)
    tables = np.full((S, W), -1, dtype=np.int64)
    k = 0
    for s, L in enumerate(lens):
        n = -(-L // B)
        tables[s, :n] = perm[k:k + n]
        k += n
    kp = rng.standard_normal((NB, Hk, B, D)).astype(np.float16)
    vp = rng.standard_normal((NB, Hk, B, D)).astype(np.float16)
    q_start = np.concatenate([[0], np.cumsum(nq)]).astype(np.int64)
    q = rng.standard_normal((int(q_start[-1]), Hq, D)).astype(np.float16)
    return q, kp, vp, tables, np.array(lens), q_start, B


def test_causal_rows_by_brute_force_loops():
    q, kp, vp, tables, lens, q_start, B = _case(1)
    out = paged_prefill(q, kp, vp, tables, lens, q_start, 0.3, B, "f16", "f16")
    Hk, g = kp.shape[1], q.shape[1] // kp.shape[1]
    for s in range(len(lens)):
        L, n = int(lens[s]), int(q_start[s + 1] - q_start[s])
        for j in range(n):
            p = L - n + j
            for i in range(q.shape[1]):
                h = i // g
                K = [[float(x) for x in kp[tables[s][t // B], h, t % B]] for t in range(p + 1)]
                V = [[float(x) for x in vp[tables[s][t // B], h, t % B]] for t in range(p + 1)]
                want = contiguous_attention_loops([float(x) for x in q[q_start[s] + j, i]], K, V, 0.3)
                assert np.allclose(out[q_start[s] + j, i], want, rtol=0, atol=1e-12)


def test_last_row_is_the_decode_step_and_first_row_a_shorter_decode():
    q, kp, vp, tables, lens, q_start, B = _case(2)
    out = paged_prefill(q, kp, vp, tables, lens, q_start, 0.25, B, "f16", "f16")
    last = q_start[1:] - 1
    dec = paged_decode(q[last], kp, vp, tables, lens, 0.25, B, "f16", "f16")
    assert np.array_equal(out[last], dec)
    first = q_start[:-1]
    n = q_start[1:] - q_start[:-1]
    dec0 = paged_decode(q[first], kp, vp, tables, lens - n + 1, 0.25, B, "f16", "f16")
    assert np.array_equal(out[first], dec0)


def test_block_placement_does_not_matter():
    q, kp, vp, tables, lens, q_start, B = _case(3)
    out = paged_prefill(q, kp, vp, tables, lens, q_start, 0.5, B, "f16", "f16")
    NB = kp.shape[0]
    perm = np.random.default_rng(9).permutation(NB)
    inv = np.argsort(perm)
    kp2, vp2 = kp[inv], vp[inv]          # block b moves to perm[b]
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    out2 = paged_prefill(q, kp2, vp2, t2, lens, q_start, 0.5, B, "f16", "f16")
    assert np.array_equal(out, out2)


def test_future_tokens_do_not_leak():
    # changing K/V at positions after a row's token leaves that row unchanged
    q, kp, vp, tables, lens, q_start, B = _case(4)
    out = paged_prefill(q, kp, vp, tables, lens, q_start, 0.5, B, "f16", "f16")
    s, L, n = 0, int(lens[0]), int(q_start[1] - q_start[0])
    blk, off = tables[s][(L - 1) // B], (L - 1) % B
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[blk, :, off] = 7
    vp2[blk, :, off] = -7
    out2 = paged_prefill(q, kp2, vp2, tables, lens, q_start, 0.5, B, "f16", "f16")
    rows_before = list(range(q_start[0], q_start[0] + n - 1))   # positions <= L - 2
    assert np.array_equal(out[rows_before], out2[rows_before])
    assert not np.array_equal(out[q_start[0] + n - 1], out2[q_start[0] + n - 1])
