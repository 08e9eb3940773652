"""BF16 field split (oracle; test infrastructure only).

*Unweight*, section "How model weights compress effectively": a BF16 number is
1 sign bit, 8 exponent bits and 7 mantissa bits.  Section "Exponents are
surprisingly predictable": the sign and mantissa are kept verbatim and only the
exponent byte is entropy coded.

Reading taken (the post gives the field widths, not a byte layout): the
verbatim byte is ``S = sign << 7 | mantissa`` (sign in bit 7, mantissa in bits
6..0), and the exponent byte is ``E = (bits >> 7) & 0xFF``.
"""
from __future__ import annotations

import numpy as np


def split_fields(w_bits: np.ndarray):
    """Return (S, E) for raw BF16 bits: S = sign<<7 | mantissa, E = exponent byte."""
    b = np.asarray(w_bits, dtype=np.uint16).astype(np.uint32)
    sign = (b >> 15) & 0x1
    exponent = (b >> 7) & 0xFF
    mantissa = b & 0x7F
    s = ((sign << 7) | mantissa).astype(np.uint8)
    return s, exponent.astype(np.uint8)


def exponent_bytes(w_bits: np.ndarray) -> np.ndarray:
    return split_fields(w_bits)[1]


def join_fields(s: np.ndarray, e: np.ndarray) -> np.ndarray:
    """Inverse of :func:`split_fields`: bits = sign<<15 | E<<7 | mantissa."""
    s32 = np.asarray(s, dtype=np.uint8).astype(np.uint32)
    e32 = np.asarray(e, dtype=np.uint8).astype(np.uint32)
    sign = (s32 >> 7) & 0x1
    mantissa = s32 & 0x7F
    return ((sign << 15) | (e32 << 7) | mantissa).astype(np.uint16)


def to_float64(bits: np.ndarray) -> np.ndarray:
    """Exact value of BF16 bits as float64 (BF16 is the top half of a float32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
