"""Length-limited canonical Huffman code of the exponent bytes (oracle; test infrastructure only).

*Unweight*, section "Exponents are surprisingly predictable": the exponent
bytes are compressed with Huffman coding (short codes for common values, long
codes for rare ones); about 2.6 bits of information per exponent.  Section
"Sharing the GPU between decode and compute": the decoder's lookup table takes
about 16 KB of shared memory.

Readings taken where the post is silent:

* Code lengths are an optimal prefix code under a length cap ``max_len``
  (default 12, so that a 2**12-entry table of 4-byte entries is 16 KB), built
  with package-merge (Larmore & Hirschberg, 1990, "A fast algorithm for optimal
  length-limited Huffman codes").  Leaves are ordered by (count ascending,
  symbol ascending); when packages are merged into the next level, an item that
  weighs the same as a package comes first.  A lone symbol gets length 1.
* Codes are canonical, assigned as in RFC 1951 section 3.2.2: by (length,
  symbol), incrementing.  The format stores the 256 lengths, not the codes.
* The stream is the codes of E in row-major (n, k) order, concatenated most
  significant bit first.  Stream bit p is bit ``31 - p % 32`` of 32-bit word
  ``p // 32``; words are stored little-endian; the word array is zero-padded to
  a multiple of 4 words (16 bytes).
* Chunks are ``chunk_syms`` consecutive symbols (the last may be shorter);
  ``off[c]`` is the absolute bit position of chunk c's first code, and
  ``off[C]`` is the total bit count, so chunk c spans ``off[c+1] - off[c]``
  bits.  Offsets are 32-bit, so a stream is at most 2**32 - 1 bits.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------- lengths ----

def package_merge_lengths(freqs, max_len: int = 12) -> np.ndarray:
    """Optimal code lengths with every length <= max_len (package-merge).

    ``freqs`` is a length-256 (or shorter) array of symbol counts; symbols with
    count 0 get length 0.  The steps: list the leaves by increasing weight; do
    ``max_len - 1`` rounds of "pair adjacent entries into packages, then merge
    the packages back into a fresh copy of the leaves by weight"; keep the
    ``2n - 2`` lightest entries of the final list; a symbol's length is the
    number of kept entries that contain it.
    """
    freqs = [int(f) for f in freqs]
    lengths = np.zeros(len(freqs), dtype=np.int64)
    symbols = [s for s, f in enumerate(freqs) if f > 0]
    n = len(symbols)
    if n == 0:
        return lengths
    if n == 1:
        lengths[symbols[0]] = 1
        return lengths
    if (1 << max_len) < n:
        raise ValueError("max_len too small for the alphabet")

    # an entry is (weight, kind, symbol-multiset); kind 0 = leaf, 1 = package
    leaves = [(freqs[s], 0, {s: 1}) for s in sorted(symbols, key=lambda s: (freqs[s], s))]
    current = list(leaves)
    for _ in range(max_len - 1):
        packages = []
        for i in range(0, len(current) - 1, 2):
            wa, _, ma = current[i]
            wb, _, mb = current[i + 1]
            merged = dict(ma)
            for s, c in mb.items():
                merged[s] = merged.get(s, 0) + c
            packages.append((wa + wb, 1, merged))
        # stable sort: leaves keep their order, packages keep theirs, and a leaf
        # precedes a package of equal weight
        current = sorted(leaves + packages, key=lambda entry: (entry[0], entry[1]))
    for _, _, multiset in current[:2 * n - 2]:
        for s, c in multiset.items():
            lengths[s] += c
    return lengths


def kraft_sum(lengths) -> float:
    return math.fsum(2.0 ** -int(l) for l in lengths if int(l) > 0)


def entropy_bits(freqs) -> float:
    f = np.asarray(freqs, dtype=np.float64)
    total = f.sum()
    p = f[f > 0] / total
    return float(-(p * np.log2(p)).sum())


def average_code_length(freqs, lengths) -> float:
    f = np.asarray(freqs, dtype=np.float64)
    return float((f * np.asarray(lengths, dtype=np.float64)).sum() / f.sum())


# ----------------------------------------------------------- canonical codes ----

def canonical_codes(lengths) -> np.ndarray:
    """RFC 1951 section 3.2.2: count codes per length, derive each length's first
    code, then hand out codes in increasing symbol order within a length."""
    lengths = [int(l) for l in lengths]
    max_bits = max(lengths) if lengths else 0
    bl_count = [0] * (max_bits + 1)
    for l in lengths:
        if l > 0:
            bl_count[l] += 1
    next_code = [0] * (max_bits + 2)
    code = 0
    for bits in range(1, max_bits + 1):
        code = (code + bl_count[bits - 1]) << 1
        next_code[bits] = code
    codes = np.zeros(len(lengths), dtype=np.int64)
    for sym, l in enumerate(lengths):
        if l > 0:
            codes[sym] = next_code[l]
            next_code[l] += 1
    return codes


# ------------------------------------------------------------------ stream ----

def encode_bitstream(symbols: np.ndarray, lengths, codes):
    """Concatenate the codes of ``symbols`` MSB-first into 32-bit words.

    Returns (words uint32, bit_positions int64 of each symbol's first bit,
    total_bits).  Written from the definition: symbol i starts at the sum of
    the lengths of the symbols before it, and bit j of its code (most
    significant first) is stream bit ``start_i + j``.
    """
    sym = np.asarray(symbols, dtype=np.int64).reshape(-1)
    lens = np.asarray(lengths, dtype=np.int64)[sym]
    if sym.size and np.any(lens == 0):
        raise ValueError("symbol without a code")
    cods = np.asarray(codes, dtype=np.int64)[sym]
    starts = np.zeros(sym.size, dtype=np.int64)
    if sym.size:
        np.cumsum(lens[:-1], out=starts[1:])
    total = int(lens.sum())
    bits = np.zeros(max(total, 1), dtype=np.uint8)
    for j in range(int(lens.max()) if sym.size else 0):
        has = lens > j
        bit = (cods[has] >> (lens[has] - 1 - j)) & 1
        bits[starts[has] + j] = bit.astype(np.uint8)
    n_words = (total + 31) // 32
    n_words_padded = ((n_words + 3) // 4) * 4
    packed = np.packbits(bits[:total], bitorder="big")
    packed = np.concatenate([packed, np.zeros(n_words_padded * 4 - packed.size, dtype=np.uint8)])
    # first stream bit = most significant bit of the big-endian word
    words = packed.view(">u4").astype(np.uint32)
    return words, starts, total


def chunk_offsets(starts: np.ndarray, total_bits: int, chunk_syms: int) -> np.ndarray:
    """off[c] = first bit of symbol c*chunk_syms; off[C] = total_bits."""
    n = starts.size
    n_chunks = (n + chunk_syms - 1) // chunk_syms
    off = np.empty(n_chunks + 1, dtype=np.int64)
    off[:n_chunks] = starts[::chunk_syms][:n_chunks]
    off[n_chunks] = total_bits
    if total_bits >= 2 ** 32:
        raise ValueError("stream longer than 2**32 - 1 bits")
    return off.astype(np.uint32)


def _decode_tables(lengths):
    lengths = [int(l) for l in lengths]
    max_bits = max(lengths)
    count = [0] * (max_bits + 1)
    for l in lengths:
        if l > 0:
            count[l] += 1
    order = sorted((l, s) for s, l in enumerate(lengths) if l > 0)
    return max_bits, count, [s for _, s in order]


def decode_chunk(words: np.ndarray, start_bit: int, n_syms: int, lengths):
    """Bit-by-bit canonical decode of ``n_syms`` symbols starting at ``start_bit``.

    ``words`` is the uint32 stream (an array, or a list of ints).

    The textbook procedure for a canonical code: read one bit at a time; after
    each bit, if the code read so far minus the first code of this length is
    below the number of codes of this length, it names a symbol (codes of one
    length are consecutive and ordered by symbol).  Returns (symbols, end_bit).
    """
    max_bits, count, sorted_syms = _decode_tables(lengths)
    w = words if isinstance(words, list) else [int(x) for x in np.asarray(words, dtype=np.uint32)]
    pos = int(start_bit)
    out = np.empty(n_syms, dtype=np.uint8)
    for i in range(n_syms):
        code = first = index = 0
        for length in range(1, max_bits + 1):
            code |= (w[pos >> 5] >> (31 - (pos & 31))) & 1
            pos += 1
            c = count[length]
            if code - first < c:
                out[i] = sorted_syms[index + code - first]
                break
            index += c
            first = (first + c) << 1
            code <<= 1
        else:
            raise ValueError("bit pattern is not a code word")
    return out, pos


def decode_bitstream(words, offsets, lengths, n_syms: int, chunk_syms: int) -> np.ndarray:
    """Decode every chunk and check that chunk c ends exactly at off[c+1]."""
    offsets = np.asarray(offsets, dtype=np.int64)
    words = [int(x) for x in np.asarray(words, dtype=np.uint32)]  # one conversion per stream
    out = np.empty(n_syms, dtype=np.uint8)
    n_chunks = offsets.size - 1
    for c in range(n_chunks):
        lo = c * chunk_syms
        cnt = min(chunk_syms, n_syms - lo)
        syms, end = decode_chunk(words, int(offsets[c]), cnt, lengths)
        if end != int(offsets[c + 1]):
            raise ValueError(f"chunk {c} ended at bit {end}, expected {int(offsets[c + 1])}")
        out[lo:lo + cnt] = syms
    return out
