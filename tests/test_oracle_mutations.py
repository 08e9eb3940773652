"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin fails.

Each case swaps one oracle routine for a subtly wrong version (a dropped term,
a wrong bit order, a transposed operand ...) and runs the pin that should catch
it.  If a pin passes with the mistake in place, the pin is too weak.
"""
import numpy as np
import pytest

import oracle
import oracle.huffman as H
import oracle.bf16 as B
import oracle.palette as P
import oracle.gemm as G
import oracle.container as Cn
import tests.test_oracle_pins as pins


def _canonical_desc_within_length(lengths):
    lengths = [int(l) for l in lengths]
    codes = np.zeros(len(lengths), np.int64)
    order = sorted(range(len(lengths)), key=lambda s: (lengths[s], -s))
    code, prev = 0, 0
    first = True
    for s in order:
        if lengths[s] == 0:
            continue
        if first:
            code, prev, first = 0, lengths[s], False
        else:
            code = (code + 1) << (lengths[s] - prev)
            prev = lengths[s]
        codes[s] = code
    return codes


def _package_merge_keep_one_more(freqs, max_len=12):
    lengths = H.package_merge_lengths.__wrapped__(freqs, max_len)  # type: ignore[attr-defined]
    nz = np.nonzero(lengths)[0]
    if nz.size > 1:
        lengths[nz[0]] += 1  # a dropped/extra package
    return lengths


def _split_sign_low(w_bits):
    b = np.asarray(w_bits, dtype=np.uint16).astype(np.uint32)
    s = (((b & 0x7F) << 1) | ((b >> 15) & 1)).astype(np.uint8)
    return s, ((b >> 7) & 0xFF).astype(np.uint8)


def _encode_lsb_first(symbols, lengths, codes):
    words, starts, total = H.encode_bitstream.__wrapped__(symbols, lengths, codes)  # type: ignore
    rev = np.array([int(f"{int(w):032b}"[::-1], 2) for w in words], dtype=np.uint32)
    return rev, starts, total


def _pack_swapped(idx):
    # plain byte packing (element 2j low, 2j+1 high) instead of the
    # per-word interleave
    idx = np.asarray(idx, dtype=np.uint8)
    return (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)


def _pack_halves_swapped(idx):
    # odd elements in the low half-word
    idx = np.asarray(idx, dtype=np.uint8)
    sw = idx.copy()
    sw[:, 0::2], sw[:, 1::2] = idx[:, 1::2], idx[:, 0::2]
    return P.pack_nibbles.__wrapped__(sw)


def _gemm_no_transpose(x_bits, w_bits):
    return B.to_float64(x_bits) @ B.to_float64(w_bits)


def _palette_ties_descending(hist):
    hist = np.asarray(hist, dtype=np.int64)
    present = [v for v in range(256) if hist[v] > 0]
    ranked = sorted(present, key=lambda v: (-int(hist[v]), -v))[:16]
    filler = (v for v in range(256) if v not in ranked)
    while len(ranked) < 16:
        ranked.append(next(filler))
    return np.array(sorted(ranked), np.uint8)


def _palette_frequency_order(hist):
    hist = np.asarray(hist, dtype=np.int64)
    present = [v for v in range(256) if hist[v] > 0]
    ranked = sorted(present, key=lambda v: (-int(hist[v]), v))[:16]
    filler = (v for v in range(256) if v not in ranked)
    while len(ranked) < 16:
        ranked.append(next(filler))
    return np.array(ranked, np.uint8)


def _tolerance_full_step(bound, y_ref, bf16_output):
    # a whole BF16 step allowed for the final rounding instead of half of one
    tol = 1e-3 * bound + 1e-6
    if bf16_output:
        tol = tol + 2.0 ** -7 * np.abs(y_ref)
    return tol


def _escape_only_if_all_outside(e, palette):
    # a row escapes only when none of its exponents is in the palette
    e = np.asarray(e, np.uint8)
    n, k = e.shape
    inpal = np.isin(e, np.asarray(palette)).reshape(n, k // 64, 64)
    return ~inpal.any(axis=2)


def _transcode_keeps_escape_ranks(e, palette, esc):
    # the escape rows keep whatever rank their in-palette exponents have
    rank = np.zeros(256, np.uint8)
    rank[np.asarray(palette, np.int64)] = np.arange(16, dtype=np.uint8)
    return rank[np.asarray(e, np.uint8)]


def _silu_wrong_sign(g_bits, u_bits):
    g, u = B.to_float64(g_bits), B.to_float64(u_bits)
    return g / (1.0 + np.exp(g)) * u


def _offsets_at_chunk_end(starts, total_bits, chunk_syms):
    # each chunk's offset taken at its last symbol instead of its first
    n = starts.size
    c = (n + chunk_syms - 1) // chunk_syms
    last = np.minimum(np.arange(c) * chunk_syms + chunk_syms - 1, n - 1)
    return np.concatenate([starts[last], [total_bits]]).astype(np.uint32)


def _decode_first_code_off_by_one(words, start_bit, n_syms, lengths):
    # the first code of each length advanced one too far
    max_bits, count, syms = H._decode_tables(lengths)
    w = [int(x) for x in np.asarray(words, np.uint32)] if not isinstance(words, list) else words
    pos, out = int(start_bit), np.empty(n_syms, np.uint8)
    for i in range(n_syms):
        code = first = index = 0
        for length in range(1, max_bits + 1):
            code |= (w[pos >> 5] >> (31 - (pos & 31))) & 1
            pos += 1
            if 0 <= code - first < count[length]:
                out[i] = syms[index + code - first]
                break
            index += count[length]
            first = (first + count[length] + 1) << 1
            code <<= 1
        else:
            raise ValueError("not a code word")
    return out, pos


def _escape_groups_column_major(e, esc):
    # groups taken K block first, then row block
    n, k = e.shape
    kbs, nbs = k // 64, (n + 127) // 128
    off, rows = [0], []
    for kb in range(kbs):
        for nb in range(nbs):
            for r in range(nb * 128, min(n, (nb + 1) * 128)):
                if esc[r, kb]:
                    rows.append(e[r, kb * 64:(kb + 1) * 64])
            off.append(len(rows))
    exp = np.array(rows, np.uint8).reshape(-1, 64) if rows else np.zeros((0, 64), np.uint8)
    return np.array(off, np.uint32), exp


def _join_mantissa_low_bits_dropped(s, e):
    # the mantissa's lowest bit lost when the fields are joined
    s32 = np.asarray(s, np.uint8).astype(np.uint32)
    e32 = np.asarray(e, np.uint8).astype(np.uint32)
    return (((s32 >> 7) << 15) | (e32 << 7) | (s32 & 0x7E)).astype(np.uint16)


def _abs_sum_without_abs(x_bits, w_bits):
    return np.abs(B.to_float64(x_bits) @ B.to_float64(w_bits).T)


def _bitmap_bits_reversed(esc):
    # row n at bit 31 - n % 32 instead of bit n % 32
    n, kb = esc.shape
    nw = 4 * ((n + 127) // 128)
    out = np.zeros((kb, nw), np.uint64)
    for r in range(n):
        out[:, r // 32] |= esc[r, :].astype(np.uint64) << np.uint64(31 - r % 32)
    return out.astype(np.uint32)


CASES = [
    ("canonical order", oracle, "canonical_codes", _canonical_desc_within_length,
     pins.test_canonical_codes_rfc1951_example),
    ("length off by one", oracle, "package_merge_lengths", _package_merge_keep_one_more,
     lambda: pins.test_package_merge_matches_brute_force(5, 3)),
    ("sign in bit 0", oracle, "split_fields", _split_sign_low,
     pins.test_field_split_definition_values),
    ("LSB-first stream", oracle, "encode_bitstream", _encode_lsb_first,
     pins.test_bitstream_hand_example),
    ("swapped nibbles", oracle, "pack_nibbles", _pack_swapped,
     pins.test_transcode_and_nibble_order),
    ("missing transpose", G, "gemm_fp64", _gemm_no_transpose,
     pins.test_gemm_matches_fsum_triple_loop),
    ("palette tie order", oracle, "build_palette", _palette_ties_descending,
     pins.test_palette_order_and_padding),
    ("palette by frequency", oracle, "build_palette", _palette_frequency_order,
     pins.test_palette_order_and_padding),
    ("index halves swapped", oracle, "pack_nibbles", _pack_halves_swapped,
     pins.test_transcode_and_nibble_order),
    ("BF16 allowance a full step", G, "tolerance", _tolerance_full_step,
     pins.test_bf16_output_tolerance_branch),
    ("escape only if all outside", Cn, "escape_rows", _escape_only_if_all_outside,
     pins.test_planted_rare_exponent_escapes_only_its_row),
    ("escape rows keep ranks", P, "transcode", _transcode_keeps_escape_ranks,
     pins.test_transcode_and_nibble_order),
    ("SiLU sign", G, "swiglu", _silu_wrong_sign, pins.test_swiglu_closed_forms),
    ("offsets at chunk end", Cn, "chunk_offsets", _offsets_at_chunk_end,
     lambda: pins.test_chunk_offsets_delimit_chunks(64)),
    ("decoder first code off by one", H, "decode_chunk", _decode_first_code_off_by_one,
     lambda: pins.test_roundtrip_lossless("normal")),
    ("escape groups column-major", Cn, "escape_storage", _escape_groups_column_major,
     pins.test_escape_group_order_hand_example),
    ("mantissa bit dropped on join", oracle, "join_fields", _join_mantissa_low_bits_dropped,
     pins.test_field_split_roundtrip_all_patterns),
    ("bound without the absolute values", G, "abs_product_sum", _abs_sum_without_abs,
     pins.test_gemm_matches_fsum_triple_loop),
    ("escape bitmap bit order", Cn, "escape_bitmap", _bitmap_bits_reversed,
     pins.test_planted_rare_exponent_escapes_only_its_row),
]


@pytest.mark.parametrize("name,mod,attr,bad,pin", CASES, ids=[c[0] for c in CASES])
def test_pin_catches_planted_mistake(monkeypatch, name, mod, attr, bad, pin):
    original = getattr(mod, attr)
    if not hasattr(original, "__wrapped__"):
        try:
            original.__wrapped__ = original  # let a mutant call the real routine
        except AttributeError:
            pass
    monkeypatch.setattr(mod, attr, bad)
    # the pins call the routine through the ``oracle`` package namespace
    if mod is not oracle and hasattr(oracle, attr):
        monkeypatch.setattr(oracle, attr, bad)
    with pytest.raises((AssertionError, ValueError)):
        pin()
