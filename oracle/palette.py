"""Exponent palette, escape rows and palette transcode (oracle; test infrastructure only).

*Unweight*, section "Exponents are surprisingly predictable": the 16 most
frequent exponents cover more than 99% of the weights of a typical layer; a
64-weight row holding any exponent outside that top-16 palette is stored
verbatim, so the hot path decides once per row instead of branching per weight.
Section "Four ways to use compressed weights": the palette form is a 4-bit
index per weight next to the verbatim sign+mantissa byte.

Readings taken where the post is silent:

* Palette order: exponents ranked by count (descending), ties broken by the
  exponent value (ascending); index 0 is the most frequent exponent.
* Fewer than 16 distinct exponents: the palette is padded with the smallest
  byte values not already present, ascending, so its 16 entries stay distinct.
* A "row" is 64 consecutive weights along K inside one output row n:
  ``W[n, 64*kb : 64*kb + 64]``.  K must be a multiple of 64.
* An escape row keeps its 64 exponent bytes verbatim (with S, that is the raw
  BF16 row).  In the transcoded index array its 64 indices are all 0.
* Nibble packing: byte j of a row of packed indices holds element 2j in its low
  nibble and element 2j+1 in its high nibble.
"""
from __future__ import annotations

import numpy as np

ROW = 64  # weights per escape row (*Unweight*, "Exponents are surprisingly predictable")
PALETTE_SIZE = 16


def exponent_histogram(e: np.ndarray) -> np.ndarray:
    """Count of each exponent byte value over the whole matrix (256 bins)."""
    return np.bincount(np.asarray(e, dtype=np.uint8).reshape(-1), minlength=256).astype(np.int64)


def build_palette(hist: np.ndarray) -> np.ndarray:
    """The 16 most frequent exponents, most frequent first (see module readings)."""
    hist = np.asarray(hist, dtype=np.int64)
    present = [v for v in range(256) if hist[v] > 0]
    ranked = sorted(present, key=lambda v: (-int(hist[v]), v))
    palette = ranked[:PALETTE_SIZE]
    filler = (v for v in range(256) if v not in palette)
    while len(palette) < PALETTE_SIZE:
        palette.append(next(filler))
    return np.array(palette, dtype=np.uint8)


def escape_rows(e: np.ndarray, palette: np.ndarray) -> np.ndarray:
    """Boolean [N, K/64]: True where the row holds an exponent not in the palette."""
    e = np.asarray(e, dtype=np.uint8)
    n, k = e.shape
    if k % ROW:
        raise ValueError("K must be a multiple of 64")
    in_palette = np.zeros(256, dtype=bool)
    in_palette[np.asarray(palette, dtype=np.int64)] = True
    outside = ~in_palette[e]
    return outside.reshape(n, k // ROW, ROW).any(axis=2)


def transcode(e: np.ndarray, palette: np.ndarray, esc: np.ndarray) -> np.ndarray:
    """Unpacked palette indices [N, K] (uint8 in 0..15): rank of E, or 0 in escape rows."""
    e = np.asarray(e, dtype=np.uint8)
    n, k = e.shape
    rank = np.zeros(256, dtype=np.uint8)
    for i, v in enumerate(np.asarray(palette, dtype=np.int64)):
        rank[v] = i
    idx = rank[e]
    idx = idx.reshape(n, k // ROW, ROW)
    idx[np.asarray(esc, dtype=bool)] = 0
    return idx.reshape(n, k)


def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """[N, K] indices -> [N, K/2] bytes: element 2j in the low nibble of byte j."""
    idx = np.asarray(idx, dtype=np.uint8)
    lo = idx[:, 0::2] & 0xF
    hi = idx[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    n, h = packed.shape
    out = np.empty((n, 2 * h), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out
