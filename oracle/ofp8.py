"""Number formats for the CPU oracle: OFP8 E4M3 and bfloat16, written out from
their published definitions.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library's
product path never calls it.

E4M3 follows the OCP 8-bit Floating Point Specification (OFP8), revision 1.0,
section 5.1 (E4M3 encoding): 1 sign bit, 4 exponent bits with bias 7, 3
mantissa bits; the all-ones exponent with all-ones mantissa is NaN and there is
no infinity; the largest finite magnitude is 1.75 * 2^8 = 448, the smallest
normal 2^-6 and the smallest subnormal 2^-9.  Conversion here is round to
nearest, ties to even, with saturation of out-of-range finite values to +-448
(the "saturating" conversion mode the specification describes).

bfloat16 is IEEE 754 binary32 with the low 16 significand bits dropped: 8
exponent bits (bias 127), 7 stored mantissa bits.  Rounding is to nearest,
ties to even, applied once to the exact input value.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_MIN_SUBNORMAL = 2.0 ** -9


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 code (uint8) as float64; NaN codes give NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.ldexp(1.0, e - 7)
    sub = sign * (m / 8.0) * 2.0 ** -6
    val = np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & (m == 0x7), np.nan, val)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round each (finite) value to the nearest E4M3 code, ties to even,
    saturating to +-448.  Input is taken exactly (float64 holds any float32)."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64) << 7
    a = np.abs(x)
    code = np.zeros(a.shape, np.int64)
    # exponent of the binade holding a: a = f * 2^ex with f in [0.5, 1)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e_unb = ex - 1                                   # a in [2^e_unb, 2^(e_unb+1))
    is_sub = a < E4M3_MIN_NORMAL
    # normal binade: 8 steps of 2^(e-3) per binade
    n_norm = np.rint(np.ldexp(a, -(e_unb - 3)))      # in [8, 16]
    carry = n_norm >= 16
    e_n = np.where(carry, e_unb + 1, e_unb)
    n_norm = np.where(carry, 8, n_norm).astype(np.int64)
    code_norm = ((e_n + 7) << 3) | (n_norm - 8)
    # subnormal range: multiples of 2^-9; 8 * 2^-9 rounds up into the first normal
    n_sub = np.rint(np.ldexp(a, 9)).astype(np.int64)  # 0..8
    code_sub = np.where(n_sub >= 8, 0x08, n_sub)
    code = np.where(is_sub, code_sub, code_norm)
    code = np.where(a >= E4M3_MAX, 0x7E, np.minimum(code, 0x7E))
    return (code | sign).astype(np.uint8)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even) in one step;
    returns float64 holding the bfloat16 values.  Finite inputs only."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e_unb = np.maximum(ex - 1, -126)        # below 2^-126 the quantum stays 2^-133
    q = np.ldexp(np.rint(np.ldexp(a, -(e_unb - 7))), e_unb - 7)
    return np.copysign(q, x)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of values already representable in bf16."""
    f = np.asarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)
