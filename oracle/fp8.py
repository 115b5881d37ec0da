"""FP8 e4m3 storage for the KV cache (oracle; test infrastructure only).

[BLOG] "How PagedAttention Powers vLLM's KV Cache", section "Where it bites": a
quantized cache stacks with paging (paging decides where a token's K/V lives, the
cache format how large it is).  The pages give no format or scale convention; the
reading taken here: each cache tensor (K, V) has one float32 scale; a value x is
stored as e4m3(x * (1/scale)) and read back as e4m3_value * scale.

e4m3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
infinities; exponent 15 with mantissa 7 is NaN; largest finite magnitude 448;
subnormals m/8 * 2^-6.  Encoding rounds to nearest, ties to even mantissa, and
saturates finite values beyond 448 to +-448 (NaN stays NaN).

Everything here is a plain table walk over the 256 codes, written from that
definition.
"""
from __future__ import annotations

import numpy as np


def e4m3_value(code: int) -> float:
    """The real value of one 8-bit code (NaN for the two NaN codes)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_CODES = np.arange(256, dtype=np.int64)
_VALUES = np.array([e4m3_value(int(c)) for c in _CODES])
# non-negative finite codes sorted by value (0x00 .. 0x7E)
_POS = np.array([c for c in range(0x80) if not np.isnan(_VALUES[c])], dtype=np.int64)
_POS_VAL = _VALUES[_POS]
MAX_FINITE = float(_POS_VAL.max())   # 448


def decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float64 values (exact)."""
    return _VALUES[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def encode_one(x: float) -> int:
    """Round one float to the nearest e4m3 code (ties to even), saturating."""
    if np.isnan(x):
        return 0x7F
    sign = 0x80 if (x < 0 or (x == 0 and np.signbit(x))) else 0
    a = min(abs(float(x)), MAX_FINITE)
    i = int(np.searchsorted(_POS_VAL, a))          # first value >= a
    if i < len(_POS_VAL) and _POS_VAL[i] == a:
        return sign | int(_POS[i])
    lo, hi = int(_POS[i - 1]), int(_POS[i])
    dlo, dhi = a - _POS_VAL[i - 1], _POS_VAL[i] - a
    if dlo < dhi:
        return sign | lo
    if dhi < dlo:
        return sign | hi
    return sign | (lo if lo % 2 == 0 else hi)       # tie: even mantissa


def encode(x: np.ndarray) -> np.ndarray:
    """Vector version of ``encode_one`` (float array -> uint8 codes)."""
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.array([encode_one(v) for v in flat], dtype=np.uint8)
    return out.reshape(np.shape(x))


def quantize(x_f32: np.ndarray, scale: float) -> np.ndarray:
    """Stored codes of float32 values for a tensor with the given scale: the value is
    multiplied (in float32) by the float32 reciprocal of the scale, then encoded."""
    inv = np.float32(1.0) / np.float32(scale)
    return encode(np.asarray(x_f32, dtype=np.float32) * inv)


def dequantize(codes: np.ndarray, scale: float) -> np.ndarray:
    """float64 values of stored codes: e4m3 value * scale."""
    return decode(codes) * float(np.float32(scale))
