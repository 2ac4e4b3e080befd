"""Pins for oracle.attention.paged_decode.

Each check ties the oracle to something other than itself: a brute-force
contiguous routine written with plain loops, closed forms, and invariants the
paging must keep (placement permutation, shared vs duplicated prefix, unused
slots never read).
"""
import math

import numpy as np
import pytest

from oracle.attention import paged_decode, contiguous_attention_loops
from oracle.numerics import decode_e4m3


def _page(K, V, lens, B, rng, num_blocks=None, poison=True):
    """Scatter contiguous per-sequence K/V [S][L, Hk, D] into a pool at random blocks."""
    S = len(lens)
    Hk, D = K[0].shape[1], K[0].shape[2]
    nb = [-(-L // B) for L in lens]
    NB = num_blocks or sum(nb) + 3
    perm = rng.permutation(NB)
    kp = np.full((NB, Hk, B, D), np.nan if poison else 0.0, dtype=np.float16)
    vp = kp.copy()
    table = np.full((S, max(nb + [1])), -1, dtype=np.int64)
    nxt = 0
    for s in range(S):
        for b in range(nb[s]):
            blk = perm[nxt]
            nxt += 1
            table[s, b] = blk
            for o in range(B):
                t = b * B + o
                if t < lens[s]:
                    kp[blk, :, o, :] = K[s][t]
                    vp[blk, :, o, :] = V[s][t]
    return kp, vp, table


def _rand_seqs(rng, lens, Hk, D):
    K = [rng.standard_normal((L, Hk, D)).astype(np.float16) for L in lens]
    V = [rng.standard_normal((L, Hk, D)).astype(np.float16) for L in lens]
    return K, V


def test_matches_bruteforce_contiguous():
    rng = np.random.default_rng(1)
    lens = [1, 5, 11, 4]
    S, Hq, Hk, D, B = 4, 6, 2, 8, 4
    g = Hq // Hk
    K, V = _rand_seqs(rng, lens, Hk, D)
    q = rng.standard_normal((S, Hq, D)).astype(np.float16)
    kp, vp, table = _page(K, V, lens, B, rng)
    scale = 1 / math.sqrt(D)
    out = paged_decode(q, kp, vp, table, lens, scale, B, "f16", "f16")
    for s in range(S):
        for i in range(Hq):
            h = i // g
            ref = contiguous_attention_loops(
                [float(x) for x in q[s, i]],
                [[float(x) for x in K[s][t, h]] for t in range(lens[s])],
                [[float(x) for x in V[s][t, h]] for t in range(lens[s])], scale)
            assert np.allclose(out[s, i], ref, rtol=0, atol=1e-12), (s, i)


def test_one_token_context_is_v0_exactly():
    rng = np.random.default_rng(2)
    K, V = _rand_seqs(rng, [1], 1, 16)
    q = rng.standard_normal((1, 1, 16)).astype(np.float16)
    kp, vp, table = _page(K, V, [1], 16, rng)
    out = paged_decode(q, kp, vp, table, [1], 0.25, 16, "f16", "f16")
    assert np.array_equal(out[0, 0], V[0][0, 0].astype(np.float64))


def test_zero_query_gives_mean_of_v():
    rng = np.random.default_rng(3)
    lens = [37]
    K, V = _rand_seqs(rng, lens, 1, 8)
    q = np.zeros((1, 1, 8), dtype=np.float16)
    kp, vp, table = _page(K, V, lens, 16, rng)
    out = paged_decode(q, kp, vp, table, lens, 1.0, 16, "f16", "f16")
    assert np.allclose(out[0, 0], V[0][:, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-14)


def test_two_token_closed_form():
    D = 4
    K = [np.zeros((2, 1, D), dtype=np.float16)]
    K[0][0, 0, 0] = 2.0                         # x0 = 0.5 * <q, k0> = 1, x1 = 0
    V = [np.array([[[1, 2, 3, 4]], [[-1, 0, 5, 8]]], dtype=np.float16)]
    q = np.array([[[1, 0, 0, 0]]], dtype=np.float16)
    rng = np.random.default_rng(4)
    kp, vp, table = _page(K, V, [2], 16, rng)
    out = paged_decode(q, kp, vp, table, [2], 0.5, 16, "f16", "f16")
    e = math.e
    expect = (e * np.array([1, 2, 3, 4]) + np.array([-1, 0, 5, 8])) / (1 + e)
    assert np.allclose(out[0, 0], expect, rtol=0, atol=1e-15)


def test_gqa_head_map():
    # Query head i reads kv head i // g: give every kv head a constant V.
    S, Hq, Hk, D, B = 1, 6, 2, 4, 4
    lens = [7]
    rng = np.random.default_rng(5)
    K = [rng.standard_normal((7, Hk, D)).astype(np.float16)]
    V = [np.stack([np.full((7, D), h + 1.0) for h in range(Hk)], axis=1).astype(np.float16)]
    q = rng.standard_normal((S, Hq, D)).astype(np.float16)
    kp, vp, table = _page(K, V, lens, B, rng)
    out = paged_decode(q, kp, vp, table, lens, 0.5, B, "f16", "f16")
    for i in range(Hq):
        assert np.allclose(out[0, i], i // 3 + 1.0, rtol=0, atol=1e-14)


def test_placement_permutation_invariant():
    rng = np.random.default_rng(6)
    lens = [33, 18, 1]
    K, V = _rand_seqs(rng, lens, 2, 8)
    q = rng.standard_normal((3, 4, 8)).astype(np.float16)
    a = paged_decode(q, *_page(K, V, lens, 8, np.random.default_rng(10)), lens, 0.3, 8, "f16", "f16")
    b = paged_decode(q, *_page(K, V, lens, 8, np.random.default_rng(11), num_blocks=40),
                     lens, 0.3, 8, "f16", "f16")
    assert np.array_equal(a, b)


def test_shared_prefix_equals_duplicated_prefix():
    rng = np.random.default_rng(7)
    B, D, Hk = 4, 8, 1
    prefix = 8                                   # two full shared blocks
    lens = [11, 14]
    K, V = _rand_seqs(rng, lens, Hk, D)
    K[1][:prefix] = K[0][:prefix]
    V[1][:prefix] = V[0][:prefix]
    q = rng.standard_normal((2, 1, D)).astype(np.float16)
    kp, vp, table = _page(K, V, lens, B, rng)          # duplicated prefix blocks
    dup = paged_decode(q, kp, vp, table, lens, 0.4, B, "f16", "f16")
    shared = table.copy()
    shared[1, :2] = table[0, :2]                        # point seq 1 at seq 0's prefix
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[table[1, :2]] = np.nan                          # its own copies are gone
    vp2[table[1, :2]] = np.nan
    sh = paged_decode(q, kp2, vp2, shared, lens, 0.4, B, "f16", "f16")
    assert np.array_equal(dup, sh)


def test_unused_slots_never_read_and_empty_context():
    rng = np.random.default_rng(8)
    lens = [0, 5, 16]
    K, V = _rand_seqs(rng, lens, 1, 8)
    q = rng.standard_normal((3, 2, 8)).astype(np.float16)
    kp, vp, table = _page(K, V, lens, 16, np.random.default_rng(1), poison=True)
    kz, vz, _ = _page(K, V, lens, 16, np.random.default_rng(1), poison=False)
    a = paged_decode(q, kp, vp, table, lens, 0.5, 16, "f16", "f16")
    b = paged_decode(q, kz, vz, table, lens, 0.5, 16, "f16", "f16")
    assert np.all(np.isfinite(a)) and np.array_equal(a, b)
    assert np.array_equal(a[0], np.zeros((2, 8)))


def test_fp8_cache_dequantises_with_per_head_scale():
    # codes 0x38 (1.0) and 0x30 (0.5): K rows make x0 = x1, so out = mean(V).
    kp = np.full((2, 2, 4, 4), 0x7F, dtype=np.uint8)
    vp = kp.copy()
    kp[1, :, :2, :] = 0x38
    vp[1, :, 0, :] = 0x38
    vp[1, :, 1, :] = 0x30
    table = np.array([[1]])
    q = np.ones((1, 2, 4), dtype=np.float16)
    vs = np.array([2.0, 4.0], dtype=np.float32)
    out = paged_decode(q, kp, vp, table, [2], 1.0, 4, "f16", "fp8_e4m3",
                       k_scale=np.array([1.0, 3.0], dtype=np.float32), v_scale=vs)
    assert np.allclose(out[0, 0], (1.0 + 0.5) / 2 * 2.0, atol=0)
    assert np.allclose(out[0, 1], (1.0 + 0.5) / 2 * 4.0, atol=0)
    assert decode_e4m3(0x38) * 3.0 == 3.0


def test_bf16_query_kind():
    rng = np.random.default_rng(9)
    lens = [6]
    K, V = _rand_seqs(rng, lens, 1, 4)
    kp, vp, table = _page(K, V, lens, 4, rng)
    qf = np.array([[[0.5, -1.0, 2.0, 0.25]]], dtype=np.float16)
    qb = np.array([[[0x3F00, 0xBF80, 0x4000, 0x3E80]]], dtype=np.uint16)  # same values as bf16 bits
    a = paged_decode(qf, kp, vp, table, lens, 0.5, 4, "f16", "f16")
    b = paged_decode(qb, kp, vp, table, lens, 0.5, 4, "bf16", "f16")
    assert np.array_equal(a, b)
