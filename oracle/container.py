"""The encoded matrix as a whole: encode, full decode, exponent-only decode,
palette transcode (oracle; test infrastructure only).

*Unweight*, section "Exponents are surprisingly predictable" (what is stored),
section "Four ways to use compressed weights" (the four things a consumer can
make of it: BF16 weights, exponent bytes, palette indices, or the palette form
prepared at load), and the untitled passage after "Sharing the GPU between
decode and compute" on one package serving distribution (Huffman) and
inference (transcoded to the palette at load).

Everything in one encoded matrix W[N, K] (K a multiple of 64):

* ``sm``       [N, K] uint8   sign+mantissa bytes, verbatim.
* ``lengths``  [256] uint8    code length of each exponent value (0 = absent).
* ``words``    uint32         the Huffman stream of E (see ``huffman``).
* ``offsets``  [C+1] uint32   chunk start bits, last entry = total bits.
* ``palette``  [16] uint8     the 16 most frequent exponents (see ``palette``).
* ``esc_bits`` [K/64, 4*ceil(N/128)] uint32: bit n%32 of word [kb, n//32] is
  set when row (n, kb) is an escape row (each K block's words are padded to a
  multiple of 4, i.e. 16 bytes per 128-row block; padding bits are 0).
* ``esc_off``  [G+1] uint32 and ``esc_exp`` [R, 64] uint8: the verbatim exponent
  bytes of the R escape rows, grouped by (n // 128, kb) with groups in
  row-major order over (n // 128, kb) and rows ascending by n inside a group;
  group g owns rows ``esc_off[g] .. esc_off[g+1]-1``.  (Reading taken: the post
  says escape rows are kept verbatim and are staged alongside the compressed
  tiles; grouping them by 128-row block and K-block lets a consumer of one
  block fetch them as one contiguous run.)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .bf16 import split_fields, join_fields
from .huffman import (package_merge_lengths, canonical_codes, encode_bitstream,
                      chunk_offsets, decode_bitstream)
from .palette import exponent_histogram, build_palette, escape_rows, transcode, pack_nibbles, ROW

ESC_GROUP_ROWS = 128


@dataclass
class Encoded:
    N: int
    K: int
    chunk_syms: int
    max_len: int
    sm: np.ndarray
    lengths: np.ndarray
    words: np.ndarray
    offsets: np.ndarray
    total_bits: int
    palette: np.ndarray
    esc: np.ndarray          # bool [N, K/64]
    esc_bits: np.ndarray
    esc_off: np.ndarray
    esc_exp: np.ndarray
    hist: np.ndarray


def escape_bitmap(esc: np.ndarray) -> np.ndarray:
    """Pack the [N, K/64] escape flags into words [K/64, 4*ceil(N/128)]."""
    n, kb = esc.shape
    nw = 4 * ((n + ESC_GROUP_ROWS - 1) // ESC_GROUP_ROWS)
    out = np.zeros((kb, nw), dtype=np.uint64)
    for r in range(n):
        out[:, r // 32] |= esc[r, :].astype(np.uint64) << np.uint64(r % 32)
    return out.astype(np.uint32)


def escape_storage(e: np.ndarray, esc: np.ndarray):
    """(esc_off, esc_exp): verbatim exponent rows grouped by (n // 128, kb)."""
    n, k = e.shape
    kbs = k // ROW
    ngroups = ((n + ESC_GROUP_ROWS - 1) // ESC_GROUP_ROWS) * kbs
    off = np.zeros(ngroups + 1, dtype=np.int64)
    rows = []
    g = 0
    for nb in range((n + ESC_GROUP_ROWS - 1) // ESC_GROUP_ROWS):
        for kb in range(kbs):
            for r in range(nb * ESC_GROUP_ROWS, min(n, (nb + 1) * ESC_GROUP_ROWS)):
                if esc[r, kb]:
                    rows.append(e[r, kb * ROW:(kb + 1) * ROW])
            g += 1
            off[g] = len(rows)
    exp = np.array(rows, dtype=np.uint8).reshape(-1, ROW) if rows else np.zeros((0, ROW), np.uint8)
    return off.astype(np.uint32), exp


def encode(w_bits: np.ndarray, chunk_syms: int = 1024, max_len: int = 12) -> Encoded:
    """Compress W[N, K] (raw BF16 bits) into the format described above."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    n, k = w_bits.shape
    if n < 1 or k < 1 or k % ROW:
        raise ValueError("need N >= 1 and K a positive multiple of 64")
    if chunk_syms % ROW or chunk_syms <= 0:
        raise ValueError("chunk_syms must be a positive multiple of 64")
    s, e = split_fields(w_bits)
    hist = exponent_histogram(e)
    lengths = package_merge_lengths(hist, max_len)
    codes = canonical_codes(lengths)
    words, starts, total = encode_bitstream(e.reshape(-1), lengths, codes)
    offsets = chunk_offsets(starts, total, chunk_syms)
    palette = build_palette(hist)
    esc = escape_rows(e, palette)
    esc_off, esc_exp = escape_storage(e, esc)
    return Encoded(N=n, K=k, chunk_syms=chunk_syms, max_len=max_len, sm=s,
                   lengths=lengths.astype(np.uint8), words=words, offsets=offsets,
                   total_bits=total, palette=palette, esc=esc, esc_bits=escape_bitmap(esc),
                   esc_off=esc_off, esc_exp=esc_exp, hist=hist)


def decode_exp(enc: Encoded) -> np.ndarray:
    """Exponent-only decode: E[N, K] from the Huffman stream (bit by bit)."""
    e = decode_bitstream(enc.words, enc.offsets, enc.lengths, enc.N * enc.K, enc.chunk_syms)
    return e.reshape(enc.N, enc.K)


def decode_full(enc: Encoded) -> np.ndarray:
    """Full decode: BF16 bits[N, K] = join(S, decoded E)."""
    return join_fields(enc.sm, decode_exp(enc))


def transcode_from_stream(enc: Encoded) -> np.ndarray:
    """Palette transcode: packed indices [N, K/2] from the Huffman stream."""
    e = decode_exp(enc)
    return pack_nibbles(transcode(e, enc.palette, enc.esc))


def rebuild_from_palette(enc: Encoded, packed: np.ndarray) -> np.ndarray:
    """BF16 bits from S, packed palette indices and the verbatim escape rows."""
    from .palette import unpack_nibbles
    idx = unpack_nibbles(packed)
    e = np.asarray(enc.palette, dtype=np.uint8)[idx]
    kbs = enc.K // ROW
    g = 0
    for nb in range((enc.N + ESC_GROUP_ROWS - 1) // ESC_GROUP_ROWS):
        for kb in range(kbs):
            rows = [r for r in range(nb * ESC_GROUP_ROWS, min(enc.N, (nb + 1) * ESC_GROUP_ROWS))
                    if enc.esc[r, kb]]
            for j, r in enumerate(rows):
                e[r, kb * ROW:(kb + 1) * ROW] = enc.esc_exp[int(enc.esc_off[g]) + j]
            g += 1
    return join_fields(enc.sm, e)
