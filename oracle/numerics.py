"""Number formats used by the layer, written from their definitions (oracle;
test infrastructure only).

* bf16: IEEE-754 binary32 with the low 16 bits dropped (8 significant bits,
  8 exponent bits).  Rounding is round-to-nearest-even, overflow to inf.
* FP8 E4M3 ("fn" flavour of the OCP 8-bit floating point specification):
  1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals
  (exponent field 0), no infinities, NaN = S.1111.111, largest finite 448.
  The activations are stored in this format per the GLM-5.3-W4A8 model card
  (table "differences from the other 4-bit releases": FP8 per-token dynamic
  activations).  Encoding rounds to nearest even and saturates finite values
  to +-448 (the conversion the FP8 tensor-core path uses); the sign of zero is
  kept, so a negative value that underflows encodes as 0x80.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BF16_MAX = float.fromhex("0x1.fep127")


def f32_round(x):
    """Round float64 values to the nearest float32 (ties to even), as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_bits_to_f64(bits):
    """Decode bf16 bit patterns (uint16/int16 array) to float64 values."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_round(x):
    """Round float64 values to the nearest bf16 value (ties to even).

    Spacing in the binade [2^E, 2^(E+1)) is 2^(E-7); below 2^-126 the spacing
    stays 2^-133 (subnormals).  Values at or above max + half a spacing
    overflow to inf.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                       # a = m * 2**ex, m in [0.5, 1)
    binade = np.maximum(ex - 1, -126)
    q = np.ldexp(1.0, binade - 7)
    with np.errstate(invalid="ignore", over="ignore"):
        v = np.rint(a / q) * q
    v = np.where(v > BF16_MAX, np.inf, v)
    v = np.where(np.isnan(x), np.nan, v)
    v = np.where(np.isinf(x), np.inf, v)
    return np.copysign(v, x)


def f64_to_bf16_bits(x):
    """bf16 bit patterns (uint16) of ``bf16_round(x)``."""
    v = bf16_round(x).astype(np.float32)      # a bf16 value is exact in float32
    return (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def e4m3_decode(codes):
    """Decode E4M3 codes (uint8) to float64 values (NaN for 0x7F/0xFF)."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    mf = c & 0x7
    normal = np.ldexp(1.0 + mf / 8.0, ef - 7)
    sub = np.ldexp(mf / 8.0, -6)
    v = np.where(ef == 0, sub, normal)
    v = np.where((ef == 15) & (mf == 7), np.nan, v)
    return sign * v


def e4m3_encode(x):
    """Encode float64 values to E4M3 codes, round-to-nearest-even, saturating.

    In the binade [2^E, 2^(E+1)) with E >= -6 the spacing is 2^(E-3); below
    2^-6 (subnormals) the spacing stays 2^-9.  A magnitude that rounds above
    448 saturates to 448.  NaN encodes as 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    finite = np.isfinite(a)
    a_f = np.where(finite, a, 0.0)
    _, ex = np.frexp(a_f)
    binade = np.maximum(ex - 1, -6)
    q = np.ldexp(1.0, binade - 3)
    v = np.rint(a_f / q) * q                  # a/q is exact (power-of-two scaling)
    v = np.minimum(v, E4M3_MAX)
    v = np.where(np.isinf(a), E4M3_MAX, v)
    # bits of the exact E4M3 value v
    _, ev = np.frexp(v)
    eb = ev - 1                               # binade of v (v > 0)
    is_sub = v < 2.0 ** -6
    mant_sub = np.rint(v / 2.0 ** -9)         # 0..7
    mant_nrm = np.rint((np.ldexp(v, -eb) - 1.0) * 8.0)
    expf = np.where(is_sub, 0, eb + 7)
    mant = np.where(is_sub, mant_sub, mant_nrm)
    bits = (expf.astype(np.int64) << 3) | mant.astype(np.int64)
    bits = np.where(neg, bits | 0x80, bits)
    bits = np.where(np.isnan(x), 0x7F, bits)
    return bits.astype(np.uint8)
