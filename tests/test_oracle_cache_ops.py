"""Pins for oracle.cache_ops on hand-built pools."""
import numpy as np

from oracle.cache_ops import reshape_and_cache, reshape_and_cache_fp8, copy_blocks, slot_of


def test_reshape_and_cache_hand_placed():
    B, Hk, D = 4, 2, 3
    kp = np.zeros((3, Hk, B, D), dtype=np.float16)
    vp = np.zeros_like(kp)
    k = np.arange(3 * Hk * D, dtype=np.float16).reshape(3, Hk, D) + 1
    v = -k
    nk, nv = reshape_and_cache(k, v, kp, vp, [5, -1, 0], B)
    exp_k = np.zeros_like(kp)
    exp_k[1, :, 1, :] = k[0]               # slot 5 = block 1, offset 1
    exp_k[0, :, 0, :] = k[2]               # slot 0 = block 0, offset 0; slot -1 skipped
    assert np.array_equal(nk, exp_k)
    assert np.array_equal(nv, -exp_k)
    assert np.array_equal(kp, np.zeros_like(kp))      # inputs untouched


def test_reshape_and_cache_fp8_codes():
    B, Hk, D = 2, 2, 4
    kp = np.full((2, Hk, B, D), 0x7F, dtype=np.uint8)
    x = np.array([[[1.0, 448.0, 1000.0, -0.0], [1.0, 0.5, -2.0, 0.0]]], dtype=np.float16)
    nk, nv = reshape_and_cache_fp8(x, x, kp, kp, [3], B, "f16",
                                   np.array([1.0, 2.0], np.float32), np.array([1.0, 0.5], np.float32))
    assert list(nk[1, 0, 1]) == [0x38, 0x7E, 0x7E, 0x80]
    assert list(nk[1, 1, 1]) == [0x30, 0x28, 0xB8, 0x00]   # x / 2: 0.5, 0.25, -1, 0
    assert list(nv[1, 1, 1]) == [0x40, 0x38, 0xC8, 0x00]   # x / 0.5: 2, 1, -4, 0
    assert np.all(nk[0] == 0x7F) and np.all(nk[1, :, 0] == 0x7F)


def test_copy_blocks_reads_pre_call_state():
    kp = np.arange(4 * 1 * 2 * 2, dtype=np.float16).reshape(4, 1, 2, 2)
    vp = kp * 10
    nk, nv = copy_blocks(kp, vp, [[0, 2], [2, 1]])
    assert np.array_equal(nk[2], kp[0]) and np.array_equal(nk[1], kp[2])
    assert np.array_equal(nk[0], kp[0]) and np.array_equal(nk[3], kp[3])
    assert np.array_equal(nv[1], vp[2])


def test_slot_of():
    assert slot_of([7, 3, 9], 40, 16) == 9 * 16 + 8     # tok 40 -> logical 2 -> phys 9
    assert slot_of([7, 3, 9], 15, 16) == 7 * 16 + 15
