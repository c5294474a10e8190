"""Exact number formats used by the oracle.  TEST INFRASTRUCTURE ONLY.

* fp16 and bf16 bit patterns are decoded exactly to float64.
* FP8-E4M3 (the OCP 8-bit "E4M3" format, no infinities) is decoded from its
  definition and encoded by round-to-nearest-even with saturation.

The FP8 KV cache is named in "KV 缓存与分页注意力", §后来的做法 (vLLM can store
the cache as 8-bit floats, one byte per number, about twice the tokens in the
same memory).  The page gives no format details; the encoding follows the
published OCP FP8 E4M3 definition:

    sign 1 bit, exponent 4 bits (bias 7), mantissa 3 bits;
    exponent field 0      -> subnormal  (-1)^s * 2^-6 * (m / 8)
    exponent field 1..15  -> normal     (-1)^s * 2^(e-7) * (1 + m / 8)
    e = 15 and m = 7      -> NaN (no infinities); largest finite value 448.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


def f16_to_f64(a: np.ndarray) -> np.ndarray:
    """IEEE binary16 values (numpy float16) -> float64, exact."""
    return np.asarray(a, dtype=np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64, exact: a bf16 value is the
    upper half of the float32 with the same sign and exponent."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Decode an array stored as ``dtype`` ("f32", "f16", "bf16", "fp8") to float64."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "f16":
        return f16_to_f64(a)
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    if dtype == "fp8":
        return e4m3_decode(a)
    raise ValueError(dtype)


def _e4m3_value(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)

# the non-negative finite codes 0x00..0x7E in increasing value order
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = E4M3_TABLE[:0x7F]


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """FP8-E4M3 codes (uint8) -> float64, exact."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float -> FP8-E4M3 code, round to nearest, ties to the even code, values
    beyond the largest finite magnitude saturate to +-448, NaN -> 0x7F.

    Written as a search over the 127 non-negative finite values: the nearest
    one wins; on a tie the code with an even last mantissa bit wins.  The sign
    is carried over unchanged (so -0.0 and negative values that round to zero
    give code 0x80).
    """
    x = np.asarray(x, dtype=np.float64)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    nan = np.isnan(flat)
    mag = np.abs(flat)
    neg = np.signbit(flat)
    # index of the first table value >= mag (table is increasing)
    hi = np.searchsorted(_POS_VALUES, np.minimum(mag, E4M3_MAX), side="left")
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = np.abs(_POS_VALUES[hi] - mag)
    d_lo = np.abs(mag - _POS_VALUES[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & ((_POS_CODES[lo] & 1) == 0))
    code = np.where(pick_lo, _POS_CODES[lo], _POS_CODES[hi])
    code = np.where(mag >= E4M3_MAX, 0x7E, code)   # saturate
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, E4M3_NAN_CODE, code)
    out[:] = code.astype(np.uint8)
    return out.reshape(x.shape)


def e4m3_quantize_for_pool(x_f32: np.ndarray, scale: float) -> np.ndarray:
    """The byte an FP8 pool stores for an input value x with per-tensor scale:
    the quotient x / scale is formed in float32 (IEEE division, round to
    nearest) and then encoded with ``e4m3_encode``.  Both the division's
    precision and the encoding's rounding fix which code is stored."""
    q = np.asarray(x_f32, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float64))
