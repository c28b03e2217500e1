"""Number formats used by the oracle: E2M1, E4M3, IEEE binary16, bfloat16, INT4.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this.

Definitions come from public format documents, not from the pages (which
only name the formats: NVFP4 and INT4 in the "SVDQuant: Absorbing Outliers
by Low-Rank Components for 4-Bit Diffusion Models" abstract; "nvfp4" with
group_size 16 in the quantization_config of the Diffusers blog's "Native
loading in Diffusers" section):

* E2M1 (FP4): OCP Microscaling Formats (MX) v1.0, element format: 1 sign,
  2 exponent bits (bias 1), 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3,
  4, 6; no infinity or NaN.
* E4M3: OCP 8-bit Floating Point specification (OFP8), E4M3 encoding:
  1 sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals, max 448,
  S.1111.111 is NaN, no infinity.
* binary16: IEEE 754-2008.
* bfloat16: the upper 16 bits of IEEE binary32 (8 significant bits).

All conversions round to nearest, ties to even, and saturate to the largest
finite magnitude where the format has no infinity ("satfinite").  Values are
carried in float64, which holds every float32 exactly.
"""
from __future__ import annotations

import numpy as np

# magnitude code -> value, E2M1 (OCP MX v1.0)
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


# --------------------------------------------------------------------- E2M1
def e2m1_decode(codes) -> np.ndarray:
    """4-bit code (bit 3 = sign) -> float64 value."""
    c = np.asarray(codes).astype(np.int64)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def e2m1_encode(v) -> np.ndarray:
    """float32 -> 4-bit code, round to nearest with ties to the even code,
    saturating at 6; the sign bit is kept, so a negative value that rounds
    to zero encodes as 0x8 (negative zero).

    Between two neighbouring grid values the rounding boundary is their
    midpoint.  The code whose lowest bit is 0 wins a tie, so the boundary is
    inclusive on the side of the odd code's neighbour:
        0 | 0.25 | 0.5 | 0.75 | 1 | 1.25 | 1.5 | 1.75 | 2 | 2.5 | 3 | 3.5 | 4 | 5 | 6
    ties:  ->0         ->1.0       ->1.0       ->2.0      ->2.0     ->4.0     ->4.0
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    mag = ((a > 0.25).astype(np.int64) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
           + (a > 2.5) + (a >= 3.5) + (a > 5.0))
    sign = np.signbit(v).astype(np.int64)
    return (mag | (sign << 3)).astype(np.uint8)


# --------------------------------------------------------------------- E4M3
def e4m3_decode(codes) -> np.ndarray:
    """8-bit E4M3 code -> float64 value (0x7F / 0xFF -> NaN)."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return np.where(s == 1, -val, val)


def e4m3_encode_satfinite(v) -> np.ndarray:
    """float32 -> E4M3 code, round to nearest even, clamp to +-448.

    For |v| in the binade [2^E, 2^(E+1)) with E >= -6 the spacing of E4M3
    values is 2^(E-3); below 2^-6 (subnormals) it is 2^-9.  The quotient by
    a power of two is exact, so rint() performs the only rounding.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                      # a = f * 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)
    q = np.ldexp(1.0, (E - 3).astype(np.int64))
    r = np.minimum(np.rint(a / q) * q, E4M3_MAX)
    # value -> bits
    _, ex2 = np.frexp(r)
    E2 = ex2 - 1
    normal = r >= 2.0 ** -6
    e_field = np.where(normal, E2 + 7, 0)
    m_field = np.where(normal, r / np.ldexp(1.0, (E2 - 3).astype(np.int64)) - 8.0, r / 2.0 ** -9)
    code = (e_field.astype(np.int64) << 3) | np.rint(m_field).astype(np.int64)
    code = np.where(r == 0, 0, code)
    sign = np.signbit(v).astype(np.int64)
    return (code | (sign << 7)).astype(np.uint8)


# --------------------------------------------------------------------- binary16 / bfloat16
def to_fp16(v) -> np.ndarray:
    """float32 -> IEEE binary16, round to nearest even (numpy's conversion)."""
    return np.asarray(v, dtype=np.float32).astype(np.float16)


def bf16_round(v) -> np.ndarray:
    """float64 -> nearest bfloat16 value (ties to even), returned as float64.

    One rounding straight from the float64 value.  bfloat16 keeps 8
    significant bits, so for |v| in [2^E, 2^(E+1)) the spacing is 2^(E-7);
    the smallest binade exponent is -126 (subnormals below)."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    E = np.maximum(ex - 1, -126)
    q = np.ldexp(1.0, (E - 7).astype(np.int64))
    return np.rint(v / q) * q


def bf16_bits(v) -> np.ndarray:
    """bfloat16-representable float64 values -> their 16-bit patterns."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------- INT4
def int4_encode(v) -> np.ndarray:
    """float32 -> signed 4-bit integer code in [-8, 7], round half to even."""
    v = np.asarray(v, dtype=np.float64)
    return np.clip(np.rint(v), -8, 7).astype(np.int8)


def pack_nibbles(codes) -> np.ndarray:
    """(rows, K) 4-bit codes -> (rows, K/2) bytes; element 2j goes to the low
    nibble of byte j, element 2j+1 to the high nibble."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    p = np.asarray(packed).astype(np.int64)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def int4_from_nibble(n) -> np.ndarray:
    n = np.asarray(n).astype(np.int64) & 0xF
    return np.where(n >= 8, n - 16, n).astype(np.int8)
