"""Number formats used by the layer, written from their definitions.

Test infrastructure only (see ``oracle/__init__.py``).

* bf16: IEEE-754 style binary format, 8 significant bits, exponent range of
  fp32 (min normal 2^-126).
* E4M3 ("fn" flavour used by NVFP4 group scales): 4 significant bits, bias 7,
  min normal 2^-6, subnormals m * 2^-9, max finite 448, no infinities.
* E2M1 (FP4 element): 2 significant bits, bias 1, values
  {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit -- the 4-bit float with "a sign
  bit, a small exponent and the rest mantissa" of [Note] "2. SVDQ-FP4".
* INT4: two's complement -8..+7, [Note] "1. INT4".

All encoders round to nearest, ties to even (the rounding rule the layer
fixes), and the E4M3 / E2M1 encoders saturate to the largest finite value
(satfinite).  The sign of a result that rounds to zero is kept (IEEE
behaviour), so -0.1 -> E2M1 code 0x8.

Parity: pinned against the format tables in ``tests/golden`` and against
torch's bf16 and float8_e4m3fn casts (tests/test_oracle_formats.py).
"""
from __future__ import annotations

import numpy as np


def round_to_format(v, p: int, emin: int, max_finite: float, satfinite: bool) -> np.ndarray:
    """Round fp64 values to a binary format with ``p`` significant bits.

    ``emin`` is the exponent of the smallest normal number; below it the
    spacing stays 2^(emin - p + 1) (gradual underflow).  Round half to even.
    Values whose rounded magnitude exceeds ``max_finite`` become +-max_finite
    when ``satfinite`` else +-inf.  The result is returned as fp64 (exact).
    """
    v0 = np.asarray(v, dtype=np.float64)
    v = v0.reshape(-1)
    out = np.zeros_like(v)
    fin = np.isfinite(v) & (v != 0)
    _, ex = np.frexp(v[fin])                   # v = m * 2^ex, 0.5 <= |m| < 1
    # the leading bit has weight 2^(ex-1); the spacing is 2^(ex-1-(p-1))
    lead = np.maximum(ex - 1, emin)
    ulp_exp = lead - (p - 1)
    q = np.ldexp(np.rint(np.ldexp(v[fin], -ulp_exp)), ulp_exp)   # rint = half-even
    big = np.abs(q) > max_finite
    q[big] = np.sign(q[big]) * (max_finite if satfinite else np.inf)
    out[fin] = q
    out[~fin] = v[~fin]                        # zeros (with sign), inf, nan pass through
    # keep the sign of values that rounded to zero
    zero = fin.copy()
    zero[fin] = q == 0
    out[zero] = np.copysign(0.0, v[zero])
    return out.reshape(v0.shape)


# ---------------------------------------------------------------- bf16
BF16_MAX = float(np.ldexp(255.0 / 128.0, 127))


def bf16_round(v) -> np.ndarray:
    """Round to bf16 (RNE), result as fp64 values."""
    return round_to_format(v, 8, -126, BF16_MAX, satfinite=False)


def bf16_bits(v) -> np.ndarray:
    """Round to bf16 (RNE) and return the 16-bit patterns."""
    f = bf16_round(v).astype(np.float32)       # exact: bf16 values are fp32 values
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    """16-bit patterns -> fp64 values."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- E4M3
E4M3_MAX = 448.0


def e4m3_round(v) -> np.ndarray:
    """Round to E4M3 (RNE, satfinite), result as fp64 values."""
    return round_to_format(v, 4, -6, E4M3_MAX, satfinite=True)


def e4m3_encode(v) -> np.ndarray:
    """Round to E4M3 and return the byte codes (sign | 4-bit exp | 3-bit mantissa)."""
    q = e4m3_round(v)
    sign = np.signbit(q).astype(np.uint8) << 7
    a = np.abs(q)
    code = np.zeros(a.shape, dtype=np.uint8)
    sub = (a > 0) & (a < 2.0 ** -6)
    code[sub] = np.rint(a[sub] / 2.0 ** -9).astype(np.uint8)          # exponent field 0
    nrm = a >= 2.0 ** -6
    m, ex = np.frexp(a[nrm])                   # a = m*2^ex, m in [0.5,1)
    e_field = (ex - 1 + 7).astype(np.int64)
    mant = np.rint((m * 2.0 - 1.0) * 8.0).astype(np.int64)             # exact after rounding
    code[nrm] = ((e_field << 3) | mant).astype(np.uint8)
    return code | sign


def e4m3_decode(code) -> np.ndarray:
    """E4M3 byte codes -> fp64 values (0x7F / 0xFF are NaN)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


# ---------------------------------------------------------------- E2M1
E2M1_MAX = 6.0
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_round(v) -> np.ndarray:
    """Round to E2M1 (RNE, satfinite), result as fp64 values."""
    return round_to_format(v, 2, 0, E2M1_MAX, satfinite=True)


def e2m1_encode(v) -> np.ndarray:
    """Round to E2M1 and return 4-bit codes (bit 3 = sign, bits 0-2 = magnitude index)."""
    q = e2m1_round(v)
    a = np.abs(q)
    # magnitude index: position in the value table (a is exactly one of them)
    idx = np.searchsorted(E2M1_VALUES, a).astype(np.uint8)
    return idx | (np.signbit(q).astype(np.uint8) << 3)


def e2m1_decode(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.uint8)
    return np.where(c & 0x8, -1.0, 1.0) * E2M1_VALUES[c & 0x7]


# ---------------------------------------------------------------- INT4
def int4_encode(v) -> np.ndarray:
    """Round half to even, clamp to [-8, 7]; return the two's complement nibble."""
    q = np.clip(np.rint(np.asarray(v, dtype=np.float64)), -8, 7).astype(np.int64)
    return (q & 0xF).astype(np.uint8)


def int4_decode(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.uint8).astype(np.int64) & 0xF
    return np.where(c >= 8, c - 16, c).astype(np.float64)


# ---------------------------------------------------------------- packing
def pack_nibbles(nib: np.ndarray) -> np.ndarray:
    """[..., K] nibbles -> [..., K/2] bytes, element 2j in the low nibble."""
    nib = np.asarray(nib, dtype=np.uint8)
    return (nib[..., 0::2] & 0xF) | ((nib[..., 1::2] & 0xF) << 4)


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] nibbles."""
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out
