"""Number formats used by the oracle, written from their definitions.

bf16: the upper 16 bits of an IEEE-754 binary32 value.

E4M3 ("FP8 E4M3FN" of the OCP 8-bit floating point specification, the FP8 type the
EagleQBSA article uses for V and for P, section "EagleQBSA量化叠加稀疏方案设计"):
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, the single
NaN pattern S.1111.111, largest finite magnitude 1.75 * 2^8 = 448, smallest
subnormal 2^-9.  Normal: (-1)^s * 2^(e-7) * (1 + m/8) for e in 1..15; subnormal:
(-1)^s * 2^-6 * (m/8).

Rounding to E4M3 here is round-to-nearest-even with saturation of out-of-range
finite magnitudes to 448 ("satfinite").  The article rounds P with a bit trick
that rounds half up (section "昇腾亲和的量化叠加稀疏Attention算子优化"); that is an
approximation of its hardware path, and the oracle takes nearest-even, the usual
definition.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = 2.0 ** -9
E4M3_MIN_NORMAL = 2.0 ** -6


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values, exactly."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 byte codes (uint8) -> float64 values; the NaN codes decode to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 codes (uint8), round to nearest even, saturating.

    The input is taken as float32 (the precision in which both the oracle and the
    kernel hold the value before it is rounded to FP8).  NaN maps to 0x7F.
    """
    xf = np.asarray(x, dtype=np.float32).astype(np.float64)
    nan = np.isnan(xf)
    neg = np.signbit(xf)
    a = np.abs(np.where(nan, 0.0, xf))
    # quantum (spacing of E4M3 values) in the binade of a; subnormal range has 2^-9
    _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
    unb = ex - 1                              # a in [2^unb, 2^(unb+1))
    unb = np.maximum(unb, -6)                 # below 2^-6 the spacing stays 2^-9
    quantum = np.exp2(unb.astype(np.float64) - 3.0)
    q = np.rint(a / quantum)                  # exact division by a power of two; rint = half-even
    val = np.minimum(q * quantum, E4M3_MAX)   # satfinite
    # encode val (exactly representable) into bits
    _, ev = np.frexp(val)
    ue = ev - 1
    is_sub = val < E4M3_MIN_NORMAL
    e_field = np.where(is_sub, 0, ue + 7)
    m_field = np.where(is_sub, np.rint(val / 2.0 ** -9), np.rint((val / np.exp2(ue.astype(np.float64)) - 1.0) * 8.0))
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(val == 0.0, 0, code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def round_to_e4m3(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest E4M3 value as float64 (encode, then decode)."""
    return e4m3_decode(e4m3_encode(x))
