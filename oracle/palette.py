"""Exponent palette, escape rows and palette transcode (oracle; test infrastructure only).

*Unweight*, section "Exponents are surprisingly predictable": the 16 most
frequent exponents cover more than 99% of the weights of a typical layer; a
64-weight row holding any exponent outside that top-16 palette is stored
verbatim, so the hot path decides once per row instead of branching per weight.
Section "Four ways to use compressed weights": the palette form is a 4-bit
index per weight next to the verbatim sign+mantissa byte.

Readings taken where the post is silent:

* Palette membership: exponents ranked by count (descending), ties broken by
  the exponent value (ascending); the first 16 are kept.
* Fewer than 16 distinct exponents: the palette is padded with the smallest
  byte values not already present, so its 16 entries stay distinct.
* Palette order: the 16 entries ascending by value; index i is the rank of the
  exponent among them.  (Exponent histograms of trained weights are unimodal,
  so the 16 most frequent usually form one run b..b+15, and then the index is
  simply e - b.)
* A "row" is 64 consecutive weights along K inside one output row n:
  ``W[n, 64*kb : 64*kb + 64]``.  K must be a multiple of 64.
* An escape row keeps its 64 exponent bytes verbatim (with S, that is the raw
  BF16 row).  In the transcoded index array its 64 indices are all 0.
* Nibble packing, per group of 8 consecutive indices of a row (4 bytes, read
  as one little-endian 32-bit word): bits 4t..4t+3 hold element 2t and bits
  16+4t..16+4t+3 hold element 2t+1 (t = 0..3).  So byte 0 holds elements 0
  (low nibble) and 2, byte 1 elements 4 and 6, byte 2 elements 1 and 3, byte 3
  elements 5 and 7: each 16-bit half of the word carries one index of each
  BF16 pair, in the pair's own lane.
"""
from __future__ import annotations

import numpy as np

ROW = 64  # weights per escape row (*Unweight*, "Exponents are surprisingly predictable")
PALETTE_SIZE = 16


def exponent_histogram(e: np.ndarray) -> np.ndarray:
    """Count of each exponent byte value over the whole matrix (256 bins)."""
    return np.bincount(np.asarray(e, dtype=np.uint8).reshape(-1), minlength=256).astype(np.int64)


def build_palette(hist: np.ndarray) -> np.ndarray:
    """The 16 most frequent exponents, ascending (see module readings)."""
    hist = np.asarray(hist, dtype=np.int64)
    present = [v for v in range(256) if hist[v] > 0]
    ranked = sorted(present, key=lambda v: (-int(hist[v]), v))
    palette = ranked[:PALETTE_SIZE]
    filler = (v for v in range(256) if v not in palette)
    while len(palette) < PALETTE_SIZE:
        palette.append(next(filler))
    return np.array(sorted(palette), dtype=np.uint8)


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
    """[N, K] indices -> [N, K/2] bytes, 8 indices per 4 bytes (see module readings)."""
    idx = np.asarray(idx, dtype=np.uint8) & 0xF
    n, k = idx.shape
    if k % 8:
        raise ValueError("K must be a multiple of 8")
    g = idx.reshape(n, k // 8, 8).astype(np.uint32)
    word = np.zeros((n, k // 8), dtype=np.uint32)
    for t in range(4):
        word |= g[:, :, 2 * t] << (4 * t)
        word |= g[:, :, 2 * t + 1] << (16 + 4 * t)
    return word.astype("<u4").view(np.uint8).reshape(n, k // 2)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of ``pack_nibbles``."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n, h = packed.shape
    word = packed.reshape(n, h // 4, 4).copy().view("<u4").reshape(n, h // 4).astype(np.uint32)
    out = np.empty((n, h // 4, 8), dtype=np.uint8)
    for t in range(4):
        out[:, :, 2 * t] = (word >> (4 * t)) & 0xF
        out[:, :, 2 * t + 1] = (word >> (16 + 4 * t)) & 0xF
    return out.reshape(n, 2 * h)
