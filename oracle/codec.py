"""Element formats E4M3 (OCP FP8 "E4M3FN") and E2M1 (FP4), from their definitions.

Test infrastructure only (see the package docstring).

Sources: the Blackwell FP4 practice page (section 1) describes E2M1 as one sign,
two exponent and one mantissa bit with non-uniform spacing, and micro-scaling
with the block scale stored in FP8; the FPSAttention page (section 2.1) names
E4M3 for FP8 quantization. The pages' range figures for FP4 are loose, so the
value sets here come from the bit-level definitions:

  E4M3: sign s, exponent e (4 bits, bias 7), mantissa m (3 bits).
        e == 0 : (-1)^s * m/8 * 2^-6            (subnormal, step 2^-9)
        e >= 1 : (-1)^s * (1 + m/8) * 2^(e-7)
        e == 15 and m == 7 : NaN (no infinities); max finite 448.
  E2M1: sign s (bit 3), exponent e (2 bits, bias 1), mantissa m (1 bit).
        e == 0 : (-1)^s * m * 0.5 ; e >= 1 : (-1)^s * (1 + m/2) * 2^(e-1)
        magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.

Encoding is round-to-nearest, ties to the even code (the code whose least
significant bit is 0), and saturating: magnitudes beyond the largest finite
value map to it. The sign is kept, so -0.0 and small negatives that round to
zero encode as the negative-zero code.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def e4m3_decode(codes) -> np.ndarray:
    """Decode E4M3 byte codes to float64 (NaN for S.1111.111)."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e2m1_decode(codes) -> np.ndarray:
    """Decode 4-bit E2M1 codes (0..15) to float64."""
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 3) & 1
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e - 1.0))
    return np.where(s == 1, -mag, mag)


# Non-negative finite magnitudes in code order; both tables are increasing.
_E4M3_POS = e4m3_decode(np.arange(0, 127))   # codes 0x00..0x7E
_E2M1_POS = e2m1_decode(np.arange(0, 8))     # codes 0..7


def _nearest_even_code(table: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """Index of the table entry nearest to ``mag`` (ties to the even index).

    ``table`` is increasing and starts at 0; ``mag`` is non-negative and at
    most ``table[-1]``.
    """
    hi = np.searchsorted(table, mag, side="left")        # table[hi] >= mag
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = mag - table[lo]
    d_hi = table[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo)


def e4m3_encode(x) -> np.ndarray:
    """Encode float values (float32 or float64) to E4M3 codes, RNE, saturating."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    mag = np.abs(x)
    nan = np.isnan(mag)
    mag = np.where(nan, 0.0, np.minimum(mag, E4M3_MAX))
    code = _nearest_even_code(_E4M3_POS, mag).astype(np.uint8)
    code = np.where(nan, np.uint8(0x7F), code).astype(np.uint8)
    return (code | np.where(neg, np.uint8(0x80), np.uint8(0))).astype(np.uint8)


def e2m1_encode(x) -> np.ndarray:
    """Encode float values to 4-bit E2M1 codes (0..15), RNE, saturating at 6."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("E2M1 has no NaN encoding")
    neg = np.signbit(x)
    mag = np.minimum(np.abs(x), E2M1_MAX)
    code = _nearest_even_code(_E2M1_POS, mag).astype(np.uint8)
    return (code | np.where(neg, np.uint8(8), np.uint8(0))).astype(np.uint8)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """Pack pairs of 4-bit codes along the last axis: element 2i in the low
    nibble of byte i, element 2i+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_e2m1`."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
