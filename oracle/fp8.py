"""FP8 E4M3 storage of the KV cache (oracle).

The pages quantise the model (LongLive review "INT8 quantised inference";
LongLive model card abstract, FP8); an FP8 KV cache is this library's
storage option, so the format comes from the OCP 8-bit floating point
specification (E4M3): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits; exponent field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN;
there is no infinity; the largest finite magnitude is 1.75 * 2^8 = 448.

Quantisation reading: per (token, head) row of D values,
scale = max|x| / 448 (scale = 1 when the row is all zeros),
code = round-to-nearest-even(x / scale) with saturation to +-448;
the stored value is decode(code) * scale.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of one E4M3 byte, from the bit fields."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """Values of all 256 codes (index = code)."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


_TABLE = e4m3_table()
_POS_CODES = np.array([c for c in range(0x7F)], dtype=np.int64)  # 0x00..0x7E, finite, >= 0
_POS_VALUES = _TABLE[_POS_CODES]


def _encode_magnitudes(mag: np.ndarray) -> np.ndarray:
    d = np.abs(mag[..., None] - _POS_VALUES)
    best = np.min(d, axis=-1, keepdims=True)
    cand = d == best
    # among equally near codes take the even one (a tie has exactly two, adjacent)
    even = cand & ((_POS_CODES % 2) == 0)
    pick = np.where(np.any(even, axis=-1, keepdims=True), even, cand)
    return _POS_CODES[np.argmax(pick, axis=-1)]


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code of each value (ties to the code with an even mantissa,
    i.e. an even code); magnitudes above 448 saturate to 448; the sign bit is
    the sign of x (so -0.0 and tiny negatives give 0x80). NaN is rejected."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.isnan(x)):
        raise ValueError("NaN input")
    mag = np.minimum(np.abs(x), E4M3_MAX).reshape(-1)
    code = np.empty(mag.shape, dtype=np.int64)
    step = 1 << 16                       # brute force over the 127 codes, in slices
    for i in range(0, mag.size, step):
        code[i:i + step] = _encode_magnitudes(mag[i:i + step])
    code = code.reshape(x.shape)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def e4m3_decode_array(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.int64) & 0xFF]


def quantize_rows(x: np.ndarray):
    """Per-row (last axis) E4M3 quantisation: returns (codes uint8, scale float64)."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    codes = e4m3_encode(x / scale[..., None])
    return codes, scale


def dequantize_rows(codes, scale) -> np.ndarray:
    return e4m3_decode_array(codes) * np.asarray(scale, dtype=np.float64)[..., None]
