"""Pins for oracle.numerics against the format definitions and a library cast."""
import math

import numpy as np
import pytest
import torch

from oracle.numerics import decode_e4m3, encode_e4m3, widen, E4M3_MAX


def test_e4m3_known_codes():
    # OCP E4M3: bias 7, 3 mantissa bits, exponent 0 subnormal, S.1111.111 NaN.
    assert decode_e4m3(0x38) == 1.0          # e=7, m=0
    assert decode_e4m3(0x39) == 1.125        # e=7, m=1
    assert decode_e4m3(0x30) == 0.5          # e=6
    assert decode_e4m3(0x7E) == 448.0        # e=15, m=6: largest finite
    assert decode_e4m3(0x08) == 2.0 ** -6    # smallest normal
    assert decode_e4m3(0x01) == 2.0 ** -9    # smallest subnormal
    assert decode_e4m3(0x07) == 7 * 2.0 ** -9
    assert decode_e4m3(0xB8) == -1.0
    assert decode_e4m3(0x00) == 0.0 and not math.copysign(1, decode_e4m3(0x00)) < 0
    assert decode_e4m3(0x80) == 0.0 and math.copysign(1, decode_e4m3(0x80)) < 0
    assert math.isnan(decode_e4m3(0x7F)) and math.isnan(decode_e4m3(0xFF))
    assert E4M3_MAX == 448.0


def test_e4m3_value_set():
    vals = decode_e4m3(np.arange(256))
    finite = vals[~np.isnan(vals)]
    assert len(finite) == 254                     # only the two NaN codes are not finite
    pos = decode_e4m3(np.arange(0x7F))
    assert np.all(np.diff(pos) > 0)               # codes 0..0x7E increase strictly
    # subnormal spacing 2^-9 below 2^-6, then 8 values per binade
    assert np.allclose(np.diff(pos[:9]), 2.0 ** -9)
    for e in range(1, 15):
        binade = pos[8 * e: 8 * e + 8]
        assert binade[0] == 2.0 ** (e - 7)
        assert np.allclose(np.diff(binade), 2.0 ** (e - 7) / 8)


def test_e4m3_round_trip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    back = encode_e4m3(decode_e4m3(codes).astype(np.float32))
    assert np.array_equal(back, codes.astype(np.uint8))


def test_e4m3_ties_to_even_and_saturation():
    cases = {
        1.0625: 0x38,       # halfway 1.0 (0x38, even) / 1.125 (0x39)
        1.1875: 0x3A,       # halfway 1.125 (0x39) / 1.25 (0x3A, even)
        1.06: 0x38, 1.07: 0x39,
        2.0 ** -10: 0x00,   # halfway 0 / 2^-9: to the even code 0
        1.5 * 2.0 ** -9: 0x02,  # halfway 2^-9 (0x01) / 2^-8 (0x02, even)
        448.0: 0x7E, 460.0: 0x7E, 1e6: 0x7E, float("inf"): 0x7E,
        -1000.0: 0xFE, float("-inf"): 0xFE,
        -1e-30: 0x80,       # underflow keeps the sign
        -0.0: 0x80,
        0.29: 0x29,         # between 0.28125 (0x29) and 0.3125 (0x2A), nearer the first
        0.3: 0x2A,          # same neighbours, nearer the second
    }
    for x, code in cases.items():
        assert int(encode_e4m3(np.float32(x))) == code, (x, hex(int(encode_e4m3(np.float32(x)))))
    assert int(encode_e4m3(np.float32("nan"))) == 0x7F


def test_e4m3_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200_000, generator=g) * 40
    x = x[x.abs() <= 448]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = encode_e4m3(x.numpy())
    assert np.array_equal(ours, ref)


def test_widen_bf16_and_f16():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x7F80, 0x3E80], dtype=np.uint16)
    assert list(widen(bits, "bf16")) == [1.0, -2.0, 0.0, float("inf"), 0.25]
    t = torch.randn(1000).to(torch.bfloat16)
    ref = t.float().numpy().astype(np.float64)
    ours = widen(t.view(torch.int16).numpy().view(np.uint16), "bf16")
    assert np.array_equal(ours, ref)
    h = np.array([1.0, -0.5, 65504.0], dtype=np.float16)
    assert list(widen(h, "f16")) == [1.0, -0.5, 65504.0]
