"""Storage-format decoding and the fp8-e4m3 encoder. Test infrastructure only.

The pages name the storage types only by size: "2 bytes for FP16/BF16, 1 byte
for FP8 / INT8" ("The KV Cache Size Equation", "PagedAttention and KV Cache
Management"), and fp8 as a lever that halves dtype_bytes ("Planning capacity
when context gets long", "KV-Cache Management and PagedAttention"). The bit
layouts below are the public format definitions:

  fp16   IEEE 754 binary16 (numpy's float16 is exactly that).
  bf16   the upper 16 bits of an IEEE 754 binary32.
  e4m3   OCP 8-bit floating point, E4M3: 1 sign, 4 exponent bits (bias 7),
         3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); no
         infinities; S.1111.111 is NaN; largest finite magnitude 448.

The encoder rounds to nearest with ties to even and saturates finite values
(and infinities) to +-448; NaN encodes as 0x7F. It works on float32 input,
the precision the quantised code is decided in (x / scale is formed in fp32).
"""
from __future__ import annotations

import numpy as np


def decode_e4m3(codes) -> np.ndarray:
    """fp64 value of each e4m3 code (any integer array in [0, 255])."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


# Every non-negative finite code with its value, in increasing order of value.
_POS_CODES = np.arange(0, 0x7F, dtype=np.int64)  # 0x00 .. 0x7E
_POS_VALUES = decode_e4m3(_POS_CODES)
assert np.all(np.diff(_POS_VALUES) > 0)
E4M3_MAX = float(_POS_VALUES[-1])  # 448


def encode_e4m3(x) -> np.ndarray:
    """uint8 code nearest to each float32 value (ties to even, saturating).

    Written as a search over the 127 representable magnitudes: find the two
    neighbours of |x|, keep the nearer one, and on an exact tie keep the one
    whose code is even.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)  # exact widening
    shape = x.shape
    x = x.reshape(-1)
    sign = np.signbit(x).astype(np.int64) << 7
    a = np.abs(x)
    out = np.empty(a.shape, dtype=np.int64)
    nan = np.isnan(a)
    big = ~nan & (a >= E4M3_MAX)
    mid = ~nan & ~big
    am = a[mid]
    hi = np.searchsorted(_POS_VALUES, am, side="left")  # first value >= |x|
    hi = np.clip(hi, 0, len(_POS_VALUES) - 1)
    lo = np.clip(hi - 1, 0, None)
    v_hi = _POS_VALUES[hi]
    v_lo = _POS_VALUES[lo]
    d_hi = v_hi - am
    d_lo = am - v_lo
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    exact = v_hi == am
    code = np.where(exact | pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    out[mid] = code
    out[big] = 0x7E
    out = out | sign
    out[nan] = 0x7F
    return out.astype(np.uint8).reshape(shape)


def widen(raw, kind: str) -> np.ndarray:
    """fp64 values of stored elements.

    kind "f16": numpy float16 array; "bf16": uint16 bit patterns;
    "fp8_e4m3": uint8 codes (the per-head scale is applied by the caller).
    """
    if kind == "f16":
        return np.asarray(raw, dtype=np.float16).astype(np.float64)
    if kind == "bf16":
        bits = np.asarray(raw, dtype=np.uint16).astype(np.uint32) << 16
        return bits.view(np.float32).astype(np.float64)
    if kind == "fp8_e4m3":
        return decode_e4m3(raw)
    raise ValueError(kind)


def to_float32(raw, kind: str) -> np.ndarray:
    """float32 values of stored 16-bit elements (exact)."""
    return widen(raw, kind).astype(np.float32)
