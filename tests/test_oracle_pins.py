"""Pins for the CPU oracle: each check compares it with something other than itself.

What fixes each value:
* BF16 field layout and values - the IEEE binary floating point definition
  (BF16 = the upper half of an IEEE binary32).
* Canonical codes - the RFC 1951 section 3.2.2 worked example (golden file).
* Code lengths - Kraft equality, brute force over all length vectors on tiny
  alphabets, equality with textbook (heap) Huffman when the cap does not bind,
  entropy bounds H <= L < H + 1.
* Bitstream - a hand-derived three-symbol example (golden file).
* Lossless claim of the method ("100% bit-exact"): decode(encode(W)) == W.
* Palette / escape - special cases whose answer is known without the oracle.
* Matmul - brute-force triple loop with math.fsum.
"""
import itertools
import heapq
import math
import os

import numpy as np
import pytest

import oracle
import synthdata
from oracle import huffman as H

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ BF16 ----

def test_field_split_definition_values():
    # 1.0 = 2^0: biased exponent 127, zero mantissa, positive
    s, e = oracle.split_fields(np.array([0x3F80], np.uint16))
    assert (int(s[0]), int(e[0])) == (0x00, 127)
    # -2.5 = -1.25 * 2^1: exponent 128, mantissa .25 -> 0x20, sign set
    s, e = oracle.split_fields(np.array([0xC020], np.uint16))
    assert (int(s[0]), int(e[0])) == (0x80 | 0x20, 128)
    # smallest subnormal 2^-133 has exponent byte 0
    assert oracle.to_float64(np.array([0x0001], np.uint16))[0] == 2.0 ** -133
    assert oracle.to_float64(np.array([0xC020], np.uint16))[0] == -2.5
    assert np.isinf(oracle.to_float64(np.array([0xFF80], np.uint16))[0])


def test_field_split_roundtrip_all_patterns():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    s, e = oracle.split_fields(allbits)
    assert np.array_equal(oracle.join_fields(s, e), allbits)
    # every (S, E) pair appears exactly once: the split is a bijection
    assert np.unique(s.astype(np.int64) * 256 + e).size == 65536


# ------------------------------------------------------- canonical codes ----

def _golden_rfc():
    rows = []
    with open(os.path.join(GOLDEN, "rfc1951_canonical.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            sym, ln, code = line.split()
            rows.append((int(sym), int(ln), code))
    return rows


def test_canonical_codes_rfc1951_example():
    rows = _golden_rfc()
    lengths = [ln for _, ln, _ in rows]
    codes = oracle.canonical_codes(lengths)
    for sym, ln, code in rows:
        assert format(int(codes[sym]), f"0{ln}b") == code


def test_canonical_codes_prefix_free_random():
    rng = np.random.default_rng(5)
    for _ in range(20):
        freqs = rng.integers(0, 1000, size=40)
        lengths = oracle.package_merge_lengths(freqs, 9)
        codes = oracle.canonical_codes(lengths)
        words = [format(int(codes[s]), f"0{int(lengths[s])}b")
                 for s in range(len(freqs)) if lengths[s] > 0]
        for a, b in itertools.permutations(words, 2):
            assert not b.startswith(a)


# ------------------------------------------------------------ code lengths ----

def _huffman_cost(freqs):
    """Textbook Huffman (binary heap): total cost = sum of merged weights."""
    h = [int(f) for f in freqs if f > 0]
    if len(h) == 1:
        return h[0]
    heapq.heapify(h)
    cost = 0
    while len(h) > 1:
        a = heapq.heappop(h)
        b = heapq.heappop(h)
        cost += a + b
        heapq.heappush(h, a + b)
    return cost


def _cost(freqs, lengths):
    return sum(int(f) * int(l) for f, l in zip(freqs, lengths))


def test_package_merge_kraft_equality_and_cap():
    rng = np.random.default_rng(1)
    for trial in range(40):
        n = int(rng.integers(2, 200))
        freqs = np.zeros(256, np.int64)
        syms = rng.choice(256, size=n, replace=False)
        freqs[syms] = rng.geometric(0.05, size=n) ** 2
        cap = int(max(math.ceil(math.log2(n)), rng.integers(8, 16)))
        lengths = oracle.package_merge_lengths(freqs, cap)
        assert lengths.max() <= cap
        assert np.all((lengths > 0) == (freqs > 0))
        assert oracle.kraft_sum(lengths) == 1.0


@pytest.mark.parametrize("n,cap", [(2, 2), (3, 2), (4, 2), (3, 3), (5, 3), (6, 3),
                                   (7, 3), (5, 4), (7, 4), (6, 5), (7, 5)])
def test_package_merge_matches_brute_force(n, cap):
    rng = np.random.default_rng(100 + 10 * n + cap)
    for _ in range(6):
        freqs = rng.integers(1, 60, size=n)
        if rng.random() < 0.5:
            freqs = rng.geometric(0.3, size=n) ** 3  # skewed: the cap binds
        best = None
        for lens in itertools.product(range(1, cap + 1), repeat=n):
            if sum(2.0 ** -l for l in lens) <= 1.0:
                c = _cost(freqs, lens)
                best = c if best is None else min(best, c)
        lengths = oracle.package_merge_lengths(freqs, cap)
        assert _cost(freqs, lengths) == best
        assert oracle.kraft_sum(lengths) <= 1.0


def test_package_merge_equals_huffman_when_cap_is_loose():
    rng = np.random.default_rng(2)
    for _ in range(30):
        n = int(rng.integers(2, 120))
        freqs = rng.integers(1, 10000, size=n)
        lengths = oracle.package_merge_lengths(freqs, n)  # n-1 bits always suffice
        assert _cost(freqs, lengths) == _huffman_cost(freqs)


def test_single_symbol_gets_length_one():
    freqs = np.zeros(256, np.int64)
    freqs[127] = 10
    lengths = oracle.package_merge_lengths(freqs, 12)
    assert lengths[127] == 1 and lengths.sum() == 1


def test_average_length_within_one_bit_of_entropy():
    w = synthdata.normal(256, 1024, 0.02, seed=3)
    e = oracle.exponent_bytes(w)
    hist = oracle.exponent_histogram(e)
    lengths = oracle.package_merge_lengths(hist, 12)
    hbits = oracle.entropy_bits(hist)
    avg = oracle.average_code_length(hist, lengths)
    assert hbits <= avg < hbits + 1.0


# ------------------------------------------------------------------ stream ----

def _golden_stream():
    vals = {}
    with open(os.path.join(GOLDEN, "bitstream_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *rest = line.split()
            vals[key] = rest
    return vals


def test_bitstream_hand_example():
    g = _golden_stream()
    symbols = np.array([int(x) for x in g["symbols"]], np.uint8)
    hist = np.bincount(symbols, minlength=256)
    lengths = oracle.package_merge_lengths(hist, 12)
    for item in g["lengths"]:
        sym, ln = item.split(":")
        assert lengths[int(sym)] == int(ln)
    codes = oracle.canonical_codes(lengths)
    words, starts, total = oracle.encode_bitstream(symbols, lengths, codes)
    assert [int(w) for w in words] == [int(x, 16) for x in g["words"]]
    off = oracle.chunk_offsets(starts, total, 64)
    assert [int(o) for o in off] == [int(x) for x in g["offsets"]]
    dec, end = oracle.decode_chunk(words, 0, symbols.size, lengths)
    assert np.array_equal(dec, symbols) and end == total


@pytest.mark.parametrize("chunk", [64, 128, 1024])
def test_chunk_offsets_delimit_chunks(chunk):
    w = synthdata.normal(48, 640, 0.02, seed=4)
    enc = oracle.encode(w, chunk_syms=chunk)
    assert enc.offsets[0] == 0 and int(enc.offsets[-1]) == enc.total_bits
    assert np.all(np.diff(enc.offsets.astype(np.int64)) > 0)
    # decode_bitstream raises unless every chunk ends exactly at the next offset
    e = oracle.decode_exp(enc)
    assert np.array_equal(e, oracle.exponent_bytes(w))
    assert enc.words.size % 4 == 0


# -------------------------------------------------------------- lossless ----

@pytest.mark.parametrize("maker", ["normal", "special", "student_t", "one_exp", "wide"])
def test_roundtrip_lossless(maker):
    if maker == "normal":
        w = synthdata.normal(64, 512, 0.02, seed=6)
    elif maker == "special":
        w = synthdata.special_values(64, 512, seed=7)
    elif maker == "student_t":
        w = synthdata.student_t(64, 512, 3.0, 0.015, seed=8)
    elif maker == "one_exp":
        w = synthdata.exponent_pattern(16, 256, [120], seed=9)
    else:  # 200 distinct exponents, long codes bounded by the cap
        w = synthdata.exponent_pattern(32, 1024, range(20, 220), seed=10)
    enc = oracle.encode(w, chunk_syms=256, max_len=12)
    assert int(enc.lengths.max()) <= 12
    assert np.array_equal(oracle.decode_full(enc), w)
    assert np.array_equal(oracle.decode_exp(enc), oracle.exponent_bytes(w))


# ----------------------------------------------------------- palette / escape ----

def test_palette_order_and_padding():
    hist = np.zeros(256, np.int64)
    hist[[130, 120, 125, 121]] = [5, 9, 9, 1]
    pal = oracle.build_palette(hist)
    # the four present exponents plus the smallest absent bytes, ascending
    assert list(pal) == list(range(0, 12)) + [120, 121, 125, 130]
    assert len(set(pal.tolist())) == 16
    # 17 present exponents: the last slot goes by count, then by the smaller
    # value (115 and 116 tie; 99 is rarer than both)
    hist = np.zeros(256, np.int64)
    hist[100:115] = 50 + np.arange(15)
    hist[[115, 116, 99]] = [7, 7, 3]
    assert list(oracle.build_palette(hist)) == list(range(100, 116))
    # a frequency order would put 114 (the most frequent) first
    hist[114] = 1000
    assert list(oracle.build_palette(hist)) == list(range(100, 116))


def test_at_most_16_exponents_means_no_escape_rows():
    for exps in ([100], list(range(110, 126))):
        w = synthdata.exponent_pattern(32, 256, exps, seed=11)
        enc = oracle.encode(w, chunk_syms=64)
        assert not enc.esc.any()
        assert enc.esc_exp.shape[0] == 0
        assert set(exps) <= set(enc.palette.tolist())


def test_planted_rare_exponent_escapes_only_its_row():
    w = synthdata.exponent_pattern(40, 512, list(range(110, 126)), seed=12)
    r, k = 33, 200
    w[r, k] = (w[r, k] & 0x807F) | (200 << 7)  # exponent 200 occurs once
    enc = oracle.encode(w, chunk_syms=128)
    expect = np.zeros_like(enc.esc)
    expect[r, k // 64] = True
    assert np.array_equal(enc.esc, expect)
    assert enc.esc_exp.shape == (1, 64)
    assert np.array_equal(enc.esc_exp[0], oracle.exponent_bytes(w)[r, 192:256])
    # bitmap word [kb, n // 32], bit n % 32
    assert enc.esc_bits[k // 64, r // 32] == (1 << (r % 32))
    assert enc.esc_bits.sum() == (1 << (r % 32))


def test_escape_group_order_hand_example():
    """Escape rows planted at known places; the storage order written out by hand:
    groups (n // 128, kb) in row-major order, rows ascending inside a group."""
    w = synthdata.exponent_pattern(256, 128, list(range(110, 126)), seed=19)
    planted = [(200, 0), (5, 1), (130, 0), (7, 1), (3, 0)]  # (row n, K block kb)
    for n, kb in planted:
        k = kb * 64 + 17
        w[n, k] = (w[n, k] & 0x807F) | (200 << 7)
    enc = oracle.encode(w, chunk_syms=64)
    # groups: (0, 0) holds row 3; (0, 1) rows 5, 7; (1, 0) rows 130, 200; (1, 1) none
    assert [int(v) for v in enc.esc_off] == [0, 1, 3, 5, 5]
    e = oracle.exponent_bytes(w)
    order = [(3, 0), (5, 1), (7, 1), (130, 0), (200, 0)]
    for i, (n, kb) in enumerate(order):
        assert np.array_equal(enc.esc_exp[i], e[n, kb * 64:(kb + 1) * 64]), (n, kb)


def test_escape_invariants_on_heavy_tails():
    w = synthdata.student_t(256, 1024, 3.0, 0.015, seed=13)
    enc = oracle.encode(w, chunk_syms=1024)
    e = oracle.exponent_bytes(w)
    inpal = np.isin(e, enc.palette).reshape(256, 16, 64)
    assert np.array_equal(enc.esc, ~inpal.all(axis=2))
    assert 0 < enc.esc.sum() < enc.esc.size


def test_transcode_and_nibble_order():
    idx = np.array([[1, 2, 3, 4, 15, 0] + [0] * 58], np.uint8)
    packed = oracle.pack_nibbles(idx)
    # group of 8: byte 0 = elements 0 | 2 << 4, byte 1 = 4 | 6 << 4,
    # byte 2 = 1 | 3 << 4, byte 3 = 5 | 7 << 4
    assert list(packed[0, :4]) == [0x31, 0x0F, 0x42, 0x00]
    # read as a little-endian word, element 2t sits at bits 4t, 2t+1 at 16+4t
    word = int.from_bytes(bytes(packed[0, :4]), "little")
    assert [(word >> (4 * t)) & 15 for t in range(4)] == [1, 3, 15, 0]
    assert [(word >> (16 + 4 * t)) & 15 for t in range(4)] == [2, 4, 0, 0]
    assert np.array_equal(oracle.unpack_nibbles(packed), idx)
    w = synthdata.student_t(128, 512, 3.0, 0.015, seed=14)
    enc = oracle.encode(w, chunk_syms=512)
    e = oracle.exponent_bytes(w)
    t = oracle.transcode(e, enc.palette, enc.esc)
    rows = t.reshape(128, 8, 64)
    assert np.all(rows[enc.esc] == 0)
    ok = ~np.repeat(enc.esc, 64, axis=1)
    assert np.array_equal(enc.palette[t][ok], e[ok])
    assert np.array_equal(oracle.transcode_from_stream(enc), oracle.pack_nibbles(t))


def test_palette_form_is_lossless():
    from oracle.container import rebuild_from_palette
    w = synthdata.student_t(300, 640, 3.0, 0.015, seed=15)  # ragged last 128-row group
    enc = oracle.encode(w, chunk_syms=64)
    packed = oracle.pack_nibbles(oracle.transcode(oracle.exponent_bytes(w), enc.palette, enc.esc))
    assert np.array_equal(rebuild_from_palette(enc, packed), w)


def test_exponent_statistics_match_the_text():
    # "the 16 most common exponents cover more than 99% of a typical layer",
    # "about 2.6 bits"
    w = synthdata.normal(1024, 1024, 0.02, seed=0)
    hist = oracle.exponent_histogram(oracle.exponent_bytes(w))
    top16 = np.sort(hist)[::-1][:16].sum() / hist.sum()
    assert top16 > 0.99
    assert 2.3 < oracle.entropy_bits(hist) < 2.9


# ------------------------------------------------------------------ matmul ----

def test_gemm_matches_fsum_triple_loop():
    rng = np.random.default_rng(16)
    for (m, n, k) in [(1, 1, 64), (3, 5, 64), (8, 16, 128), (2, 7, 192)]:
        x = synthdata.activations(m, k, seed=int(rng.integers(1 << 30)))
        w = synthdata.normal(n, k, 0.02, seed=int(rng.integers(1 << 30)))
        y = oracle.gemm_fp64(x, w)
        b = oracle.abs_product_sum(x, w)
        xf = oracle.to_float64(x)
        wf = oracle.to_float64(w)
        for i in range(m):
            for j in range(n):
                exact = math.fsum(xf[i, t] * wf[j, t] for t in range(k))
                assert abs(y[i, j] - exact) <= 1e-12 * b[i, j] + 1e-300
                assert y[i, j] == pytest.approx(oracle.gemm_entry_fsum(x, w, i, j), rel=1e-12,
                                                abs=1e-300)
                assert b[i, j] == pytest.approx(math.fsum(abs(xf[i, t] * wf[j, t])
                                                          for t in range(k)), rel=1e-12)


def test_tolerance_rejects_transposed_operand():
    x = synthdata.activations(64, 64, seed=17)
    w = synthdata.normal(64, 64, 0.02, seed=18)
    y = oracle.gemm_fp64(x, w)
    b = oracle.abs_product_sum(x, w)
    assert oracle.within_tolerance(y.astype(np.float32), y, b)[0]
    wrong = oracle.to_float64(x) @ oracle.to_float64(w)  # forgot the transpose
    assert not oracle.within_tolerance(wrong, y, b)[0]


def test_bf16_output_tolerance_branch():
    """The BF16-output allowance covers the one final rounding to BF16 and no
    more.  Exact sums are built from BF16 values with every product of one
    sign (so sum |x w| = |y|, and the accumulation term is 1e-3 |y|):
    round-to-nearest-even passes, rounding the wrong way or landing one BF16
    step off fails.  (A BF16 step at y in [2^e, 2^(e+1)) is 2^(e-7).)"""
    def bits(vals):
        return synthdata.to_bf16_bits(np.array(vals, np.float32)).reshape(1, -1)

    # y = 1 + 3 * 2^-9: between the BF16 values 1 and 1 + 2^-7, nearer the latter
    x = bits([1.0, 1.0, 1.0] + [0.0] * 61)
    w = bits([1.0, 2.0 ** -8, 2.0 ** -9] + [0.0] * 61)
    y_ref = oracle.gemm_fp64(x, w)
    b = oracle.abs_product_sum(x, w)
    assert y_ref[0, 0] == 1.0 + 3 * 2.0 ** -9 and b[0, 0] == y_ref[0, 0]
    ok = lambda y: oracle.within_tolerance(np.array([[y]]), y_ref, b, bf16_output=True)[0]
    assert ok(1.0 + 2.0 ** -7)            # nearest BF16
    assert not ok(1.0)                    # rounded the wrong way (3 * 2^-9 off)
    assert not ok(1.0 + 2.0 ** -6)        # one BF16 step above the right answer
    # y = 1.5 exactly representable: itself passes, one step (2^-7) either side fails
    x1 = bits([1.0, 1.0] + [0.0] * 62)
    w1 = bits([1.0, 0.5] + [0.0] * 62)
    y1, b1 = oracle.gemm_fp64(x1, w1), oracle.abs_product_sum(x1, w1)
    assert y1[0, 0] == 1.5
    ok1 = lambda y: oracle.within_tolerance(np.array([[y]]), y1, b1, bf16_output=True)[0]
    assert ok1(1.5)
    assert not ok1(1.5 + 2.0 ** -7) and not ok1(1.5 - 2.0 ** -7)
    # the FP32-output rule has no rounding allowance: 1 + 2^-7 fails there too
    assert not oracle.within_tolerance(np.array([[1.0 + 2.0 ** -7]]), y_ref, b)[0]


def test_synthetic_row_prefix_is_stable():
    a = synthdata.workload("gate_14336x4096", rows=8)
    b = synthdata.normal(32, 4096, 0.02, seed=10)[:8]
    assert np.array_equal(a, b)


def test_swiglu_closed_forms():
    g = synthdata.to_bf16_bits(np.array([0.0, 1.0, -1.0, 8.0, -8.0, 2.0], np.float32))
    u = synthdata.to_bf16_bits(np.array([5.0, 1.0, 1.0, 1.0, 1.0, 0.0], np.float32))
    h = oracle.swiglu(g, u)
    assert h[0] == 0.0                                  # SiLU(0) = 0
    assert h[1] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)  # sigmoid(1)
    assert h[1] - h[2] == pytest.approx(1.0, rel=1e-15)  # SiLU(x) - SiLU(-x) = x
    assert h[3] == pytest.approx(8.0, rel=1e-3) and abs(h[4]) < 3e-3  # tails -> x and 0
    assert h[5] == 0.0                                  # u = 0
