"""The decoders' lookup tables, built on the host, checked entry by entry (no GPU).

The library builds one 2^12-entry table per matrix from the code lengths and
the palette (the post's ~16 KB decoder table, *Unweight* section "Sharing the
GPU between decode and compute"), plus canonical-code tables for decoding one
code at a time.  Each entry describes the 12-bit window of stream bits it is
indexed by:

* bits 0..3: stream bits the entry consumes; bits 4..8: 4 x symbols it yields;
* bit 9 (special): the window starts with the code of an exponent outside the
  palette, or with no code at all (bit 10 too); one placeholder rank 0 is
  yielded and the code's length (1 bit without a code) consumed;
* bits 12..31: the palette ranks of the whole codes at the window's start, at
  most five, stopping before a code of an exponent outside the palette.

Here every entry of the library's table is compared with a parse of its window
by the oracle's canonical code (RFC 1951 section 3.2.2), and streams encoded by
the oracle are decoded through the tables the way the decoders use them.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import synthdata

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT_BITS = 12
MAX_RANKS = 5
SPECIAL, INVALID = 1 << 9, 1 << 10
CANON_LIMIT, CANON_FIRST, CANON_OFFSET, CANON_SYMBOLS = 0, 16, 32, 48


@pytest.fixture(scope="module")
def dump_tool(tmp_path_factory):
    exe = tmp_path_factory.mktemp("lut") / "lut_dump"
    csrc = os.path.join(ROOT, "decode_gemm_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", os.path.join(ROOT, "include"),
                    "-I", csrc, os.path.join(ROOT, "tests", "lut_dump.cpp"),
                    os.path.join(csrc, "encode.cpp"), "-o", str(exe)], check=True)
    return str(exe)


def _library_tables(tool, lengths, palette):
    text = " ".join(str(int(v)) for v in list(lengths) + list(palette))
    out = subprocess.run([tool], input=text, capture_output=True, text=True, check=True).stdout
    vals = [int(v) for v in out.split()]
    if vals[0] != 1:
        return None
    lut = np.array(vals[1:1 + (1 << LUT_BITS)], dtype=np.int64)
    canon = np.array(vals[1 + (1 << LUT_BITS):], dtype=np.int64)
    return lut, canon


def _code_map(lengths):
    codes = oracle.canonical_codes(lengths)
    return {(int(lengths[s]), int(codes[s])): s for s in range(256) if lengths[s]}


def _first_code(window, cmap, n_bits=LUT_BITS):
    """(symbol, length) of the code that starts the window, or None."""
    for l in range(1, n_bits + 1):
        s = cmap.get((l, window >> (n_bits - l)))
        if s is not None:
            return s, l
    return None


def _expected_entry(window, cmap, rank):
    first = _first_code(window, cmap)
    if first is None:
        return {"bits": 1, "count": 1, "special": True, "invalid": True, "ranks": [0]}
    if rank[first[0]] < 0:
        return {"bits": first[1], "count": 1, "special": True, "invalid": False, "ranks": [0]}
    ranks, used = [], 0
    while len(ranks) < MAX_RANKS and used < LUT_BITS:
        rest = (window << used) & ((1 << LUT_BITS) - 1)
        nxt = _first_code(rest, cmap)
        if nxt is None or rank[nxt[0]] < 0 or used + nxt[1] > LUT_BITS:
            break
        ranks.append(rank[nxt[0]])
        used += nxt[1]
    return {"bits": used, "count": len(ranks), "special": False, "invalid": False, "ranks": ranks}


def _fields(e):
    count = ((e >> 4) & 31) // 4
    return {"bits": e & 15, "count": count, "special": bool(e & SPECIAL),
            "invalid": bool(e & INVALID),
            "ranks": [(e >> (12 + 4 * i)) & 15 for i in range(count)]}


def _first_code_len(canon, window):
    l = 1
    while l < LUT_BITS and window >= canon[CANON_LIMIT + l]:
        l += 1
    return l


def _canon_symbol(canon, window):
    l = _first_code_len(canon, window)
    k = canon[CANON_OFFSET + l] + (window >> (LUT_BITS - l)) - canon[CANON_FIRST + l]
    syms = canon[CANON_SYMBOLS:].astype("<u4").tobytes()
    return syms[int(k) & 255], l


def _cases():
    """(name, histogram, code-length cap): the synthetic workloads' exponent
    statistics, tiny and skewed alphabets, palettes that are and are not one
    run, codes that use the whole 12-bit cap, and an incomplete code."""
    out = []
    for name, w in [("normal", synthdata.normal(256, 1024, 0.02, seed=401)),
                    ("student_t", synthdata.student_t(256, 1024, 3.0, 0.015, seed=402)),
                    ("special_values", synthdata.special_values(64, 1024, seed=403))]:
        out.append((name, oracle.exponent_histogram(oracle.exponent_bytes(w)), 12))
    h = np.zeros(256, np.int64)
    h[127] = 1000
    out.append(("one exponent (incomplete code)", h, 12))
    h = np.zeros(256, np.int64)
    h[[3, 90, 200]] = [5, 7, 11]
    out.append(("three far-apart exponents", h, 12))
    rng = np.random.default_rng(404)
    h = np.zeros(256, np.int64)
    sup = rng.choice(256, size=40, replace=False)
    h[sup] = rng.integers(1, 10**6, size=40)
    out.append(("40 scattered exponents (palette not a run)", h, 12))
    h = np.zeros(256, np.int64)
    h[100:140] = (2.0 ** -np.arange(40) * 2**40).astype(np.int64) + 1
    out.append(("geometric counts (lengths at the cap)", h, 12))
    out.append(("geometric counts, cap 6", h, 6))
    h = np.zeros(256, np.int64)
    h[110:126] = rng.integers(1, 1000, size=16)
    out.append(("16 exponents, no escapes", h, 12))
    return out


CASES = _cases()


@pytest.mark.parametrize("name,hist,cap", CASES, ids=[c[0] for c in CASES])
def test_every_table_entry(dump_tool, name, hist, cap):
    lengths = oracle.package_merge_lengths(hist, cap)
    palette = oracle.build_palette(hist)
    tables = _library_tables(dump_tool, lengths, palette)
    assert tables is not None
    lut, canon = tables
    cmap = _code_map(lengths)
    rank = np.full(256, -1)
    rank[palette] = np.arange(16)
    n_special = 0
    for window in range(1 << LUT_BITS):
        want = _expected_entry(window, cmap, rank)
        got = _fields(int(lut[window]))
        assert got == want, (window, got, want)
        n_special += want["special"]
        first = _first_code(window, cmap)
        if first is not None:  # the one-code-at-a-time tables agree
            assert _first_code_len(canon, window) == first[1], window
            assert _canon_symbol(canon, window) == first, window
    if name.startswith("one exponent"):
        assert n_special == 1 << (LUT_BITS - 1)  # windows starting with a 1: no code


def _table_decode(lut, canon, palette, words, start, n_syms):
    """Decode n_syms symbols from stream bit `start` through the tables: whole
    entries while they fit the symbols left, the first code alone otherwise;
    a special entry's exponent comes from the canonical tables.  Returns the
    exponents and the bit position reached."""
    bits = np.unpackbits(words.astype(">u4").view(np.uint8))
    bits = np.concatenate([bits, np.zeros(LUT_BITS, np.uint8)])
    pos, out = start, []
    while len(out) < n_syms:
        window = int("".join(map(str, bits[pos:pos + LUT_BITS])), 2)
        e = int(lut[window])
        f = _fields(e)
        if f["count"] > n_syms - len(out):
            f = {"bits": _first_code_len(canon, window), "count": 1, "special": False,
                 "invalid": False, "ranks": f["ranks"][:1]}
        assert not f["invalid"], pos
        if f["special"]:
            sym, l = _canon_symbol(canon, window)
            assert l == f["bits"]
            out.append(sym)
        else:
            out.extend(int(palette[r]) for r in f["ranks"])
        pos += f["bits"]
    return np.array(out), pos


@pytest.mark.parametrize("name,hist,cap", CASES[:3] + CASES[4:7], ids=[c[0] for c in CASES[:3] + CASES[4:7]])
def test_streams_decode_through_the_tables(dump_tool, name, hist, cap):
    lengths = oracle.package_merge_lengths(hist, cap)
    palette = oracle.build_palette(hist)
    lut, canon = _library_tables(dump_tool, lengths, palette)
    rng = np.random.default_rng(405)
    support = np.flatnonzero(hist)
    p = hist[support] / hist[support].sum()
    sym = rng.choice(support, size=1500, p=p)
    sym[::97] = rng.choice(support, size=sym[::97].size)  # rare exponents too
    codes = oracle.canonical_codes(lengths)
    words, starts, total = oracle.encode_bitstream(sym, lengths, codes)
    chunk = 128
    offsets = oracle.chunk_offsets(starts, total, chunk)
    for c in range(offsets.size - 1):
        n = min(chunk, sym.size - c * chunk)
        got, end = _table_decode(lut, canon, palette, words, int(offsets[c]), n)
        assert np.array_equal(got, sym[c * chunk:c * chunk + n]), c
        assert end == offsets[c + 1], c  # each chunk ends exactly at the next offset


def test_tables_refused_for_codes_the_table_cannot_hold(dump_tool):
    lengths = np.zeros(256, np.uint8)
    lengths[[1, 2]] = [1, 13]  # longer than the 12-bit window
    assert _library_tables(dump_tool, lengths, np.arange(16)) is None
    lengths[[1, 2, 3]] = [1, 1, 1]  # Kraft sum above 1
    assert _library_tables(dump_tool, lengths, np.arange(16)) is None
