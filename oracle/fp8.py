"""Oracle FP8 (e4m3) storage of the KV cache.

TEST INFRASTRUCTURE (see oracle/__init__.py).

"vLLM PagedAttention 深度解析" §7.4 (FP8 KV cache): K and V are stored as 8-bit
floats so a block holds twice the tokens. The pages name no format details;
readings taken here:
- the format is e4m3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
  bits; no infinities; S.1111.111 is NaN; largest finite value 448 =
  1.75 * 2^8; subnormals m * 2^-9);
- one scale per tensor (K and V each): a value x is stored as
  e4m3(float32(x * inv_scale)) with inv_scale = float32(1 / scale), rounded to
  nearest, ties to even, and values beyond the largest finite magnitude
  saturate to +-448; the cache value it stands for is decode(code) * scale.

Written from the format's definition: encode walks the exponent range and
rounds the significand; decode assembles sign, exponent and mantissa.
"""
from __future__ import annotations

import math

import numpy as np

MAX_E4M3 = 448.0
_BIAS = 7


def decode(code: int) -> float:
    """Value of one e4m3 code (0..255)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * m * 2.0 ** (1 - _BIAS - 3)          # subnormal: m/8 * 2^-6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - _BIAS)


_TABLE = np.array([decode(c) for c in range(256)], dtype=np.float64)


def decode_array(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def _round_half_even(x: float) -> int:
    f = math.floor(x)
    r = x - f
    if r > 0.5 or (r == 0.5 and f % 2 == 1):
        return int(f) + 1
    return int(f)


def encode(x: float) -> int:
    """e4m3 code of x: round to nearest, ties to even; |x| beyond 448 gives
    +-448 (saturation); NaN gives 0x7F."""
    x = float(x)
    if math.isnan(x):
        return 0x7F
    sign = 0x80 if (x < 0 or (x == 0 and math.copysign(1.0, x) < 0)) else 0
    a = abs(x)
    if a == 0:
        return sign
    if a > MAX_E4M3 * 2:                                  # far beyond the range (incl. infinity)
        return sign | 0x7E
    # quantum (distance between neighbours) at a's binade; subnormals share 2^-9
    e = max(math.floor(math.log2(a)), 1 - _BIAS)
    # guard against log2 rounding at binade edges
    while a >= 2.0 ** (e + 1):
        e += 1
    while e > 1 - _BIAS and a < 2.0 ** e:
        e -= 1
    q = 2.0 ** (e - 3)
    n = _round_half_even(a / q)                           # significand in units of q
    if n == 16:                                           # rounded up into the next binade
        e, n = e + 1, 8
    value = n * q
    if value > MAX_E4M3:
        return sign | 0x7E
    if e == 1 - _BIAS and n < 8:
        return sign | n                                   # subnormal (or rounded to 0)
    return sign | ((e + _BIAS) << 3) | (n - 8)


def encode_array(x) -> np.ndarray:
    """encode() applied elementwise, written with array operations: the binade
    from frexp (subnormals share the lowest binade's quantum 2^-9), the
    significand rounded half to even (np.rint), a carry into the next binade,
    then saturation, zeros, signs and NaN as in encode()."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(a)
        e = np.maximum(e.astype(np.int64) - 1, 1 - _BIAS)        # floor(log2 a), at least -6
        n = np.rint(a / np.ldexp(1.0, e - 3))                    # significand in quanta
        carry = n >= 16
        e = np.where(carry, e + 1, e)
        n = np.where(carry, 8, n)
        value = n * np.ldexp(1.0, e - 3)
        sat = ~(value <= MAX_E4M3) | np.isinf(a)                # beyond 448, infinity
    n = np.where(np.isfinite(n), n, 0).astype(np.int64)
    sub = (e == 1 - _BIAS) & (n < 8)
    code = np.where(sub, n, ((e + _BIAS) << 3) | np.maximum(n - 8, 0))
    code = np.where(sat, 0x7E, code)
    code = np.where(a == 0, 0, code)
    code = code | (np.signbit(x).astype(np.int64) << 7)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize(x, scale: float) -> np.ndarray:
    """Codes stored for x under a per-tensor scale: encode(float32(x * inv)),
    inv = float32(1 / scale), products and the reciprocal in float32."""
    inv = np.float32(1.0) / np.float32(scale)
    return encode_array(np.asarray(x, dtype=np.float32) * inv)


def dequantize(codes, scale: float) -> np.ndarray:
    """The cache values the codes stand for (fp64): decode(code) * scale."""
    return decode_array(codes) * float(np.float32(scale))
