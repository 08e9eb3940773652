"""CPU tests of the C-ABI library: exports, host encoder == oracle, validation.

No GPU is needed: the host encoder and the format validator are host code.
Device entry points are only checked for being exported here.
"""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import synthdata

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def uw():
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200
    return decode_gemm_b200


def _header_text():
    text = open(os.path.join(ROOT, "include", "unweight.h")).read()
    return re.sub(r"/\*.*?\*/", "", text, flags=re.S)


def _declared_functions():
    return sorted(set(re.findall(r"\b(uw_[a-z0-9_]+)\s*\(", _header_text())))


def test_library_exports_every_declared_symbol(uw):
    declared = _declared_functions()
    assert len(declared) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", uw.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (uw_\w+)", out))
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    # nothing exported that the header does not declare
    assert exported <= set(declared), sorted(exported - set(declared))
    for name in declared:
        assert hasattr(uw.lib, name)


def test_binding_constants_match_header(uw):
    """Status codes, pipeline ids and trace kinds in the binding are the header's values."""
    vals = {n: int(v) for n, v in re.findall(r"\b(UW_[A-Z0-9_]+)\s*=\s*(\d+)", _header_text())}
    status = [n for n in vals if n == "UW_OK" or n.startswith("UW_ERR_")]
    pipes = [n for n in vals if n.startswith("UW_PIPE_")]
    kinds = [n for n in vals if n.startswith("UW_KERNEL_")]
    assert len(status) == 11 and len(pipes) == 6 and len(kinds) == 11
    for n in status + pipes:
        assert getattr(uw, n) == vals[n], n
    assert len(uw.KERNEL_KINDS) == len(kinds)
    for n in kinds:
        assert uw.KERNEL_KINDS[vals[n]] == n[len("UW_KERNEL_"):].lower(), n


_STRUCTS = ("uw_encode_opts", "uw_format", "uw_stats_t", "uw_gemm_config", "uw_mlp_layer",
            "uw_mlp_opts")


def test_binding_structs_match_header(uw, tmp_path):
    """Each ctypes mirror has the C compiler's size and field offsets for the header's struct."""
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "unweight.h"', "int main(void) {"]
    for s in _STRUCTS:
        lines.append(f'  printf("{s} %zu\\n", sizeof({s}));')
        for f, _ in getattr(uw, s)._fields_:
            lines.append(f'  printf("{s}.{f} %zu %zu\\n", offsetof({s}, {f}), '
                         f"sizeof((({s}*)0)->{f}));")
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True)
    got = dict(l.split(" ", 1) for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                      check=True).stdout.splitlines())
    for s in _STRUCTS:
        cls = getattr(uw, s)
        assert int(got[s]) == C.sizeof(cls), s
        for f, t in cls._fields_:
            off, size = map(int, got[f"{s}.{f}"].split())
            assert (off, size) == (getattr(cls, f).offset, C.sizeof(t)), (s, f)


def test_status_strings(uw):
    assert uw.uw_status_str(uw.UW_OK) == "ok"
    for s in range(1, 10):
        assert uw.uw_status_str(s) not in ("", "unknown status")
    assert uw.uw_status_str(99) == "unknown status"
    assert uw.lib.uw_abi_version() == 1


def _compare_with_oracle(uw, w, chunk, max_len=12):
    h = uw.uw_encode_host(w, uw.default_opts(chunk_syms=chunk, max_code_len=max_len))
    a = h.arrays()
    ref = oracle.encode(w, chunk_syms=chunk, max_len=max_len)
    assert np.array_equal(a["code_len"], ref.lengths)
    assert np.array_equal(a["palette"], ref.palette)
    assert np.array_equal(a["words"], ref.words)
    assert np.array_equal(a["chunk_off"], ref.offsets)
    assert np.array_equal(a["sm"], ref.sm.reshape(-1))
    assert np.array_equal(a["esc_bits"], ref.esc_bits.reshape(-1))
    assert np.array_equal(a["esc_off"], ref.esc_off)
    assert np.array_equal(a["esc_exp"], ref.esc_exp.reshape(-1))
    return h, ref


@pytest.mark.parametrize("case", ["normal", "special", "student_t", "one_exp", "wide", "ragged"])
def test_host_encoder_matches_oracle(uw, case):
    if case == "normal":
        w, chunk = synthdata.normal(256, 1024, 0.02, seed=21), 1024
    elif case == "special":
        w, chunk = synthdata.special_values(128, 512, seed=22), 256
    elif case == "student_t":
        w, chunk = synthdata.student_t(300, 640, 3.0, 0.015, seed=23), 128
    elif case == "one_exp":
        w, chunk = synthdata.exponent_pattern(40, 128, [127], seed=24), 64
    elif case == "wide":
        w, chunk = synthdata.exponent_pattern(64, 512, range(0, 256), seed=25), 512
    else:  # N*K not a multiple of the chunk: short last chunk
        w, chunk = synthdata.normal(33, 192, 0.02, seed=26), 1024
    h, ref = _compare_with_oracle(uw, w, chunk)
    # the oracle's bit-by-bit decoder reads the library's stream back to W
    a = h.arrays()
    e = oracle.decode_bitstream(a["words"], a["chunk_off"], a["code_len"], w.size, chunk)
    assert np.array_equal(oracle.join_fields(a["sm"], e).reshape(w.shape), w)


def test_host_encoder_matches_oracle_at_full_gate_shape(uw):
    # the whole 14336x4096 projection: streams must be byte-identical
    w = synthdata.workload("gate_14336x4096")
    h, ref = _compare_with_oracle(uw, w, 1024)
    st = h.stats()
    assert st["max_len_used"] <= 12
    assert 2.5 < st["bits_per_exponent"] < 2.7
    assert st["top16_coverage"] > 0.99


def test_host_encoder_caps_code_length(uw):
    w = synthdata.exponent_pattern(64, 1024, range(0, 256), seed=27)
    for cap in (8, 9, 12):
        h, ref = _compare_with_oracle(uw, w, 256, max_len=cap)
        assert h.arrays()["code_len"].max() <= cap


def test_host_encoder_argument_errors(uw):
    w = synthdata.normal(4, 128, 0.02, seed=1)
    out = C.c_void_p()
    assert uw.lib.uw_encode_host(None, 4, 128, None, C.byref(out)) == uw.UW_ERR_ARG
    assert uw.lib.uw_encode_host(w.ctypes.data, 4, 100, None, C.byref(out)) == uw.UW_ERR_SHAPE
    assert uw.lib.uw_encode_host(w.ctypes.data, 0, 128, None, C.byref(out)) == uw.UW_ERR_SHAPE
    assert uw.lib.uw_encode_host(w.ctypes.data, 4, 0, None, C.byref(out)) == uw.UW_ERR_SHAPE
    bad = uw.default_opts(chunk_syms=100)
    assert uw.lib.uw_encode_host(w.ctypes.data, 4, 128, C.byref(bad), C.byref(out)) == uw.UW_ERR_ARG
    bad = uw.default_opts(max_code_len=13)
    assert uw.lib.uw_encode_host(w.ctypes.data, 4, 128, C.byref(bad), C.byref(out)) == uw.UW_ERR_ARG
    assert uw.lib.uw_validate_format(None) == uw.UW_ERR_ARG


# ------------------------------------------------ validation / fault injection --

def _buffers(uw, arrays, **over):
    a = dict(arrays)
    a.update(over)
    return uw.FormatBuffers(a["N"], a["K"], a["max_code_len"], a["chunk_syms"], a["code_len"],
                            a["palette"], a["words"], a["chunk_off"], a["sm"], a["esc_bits"],
                            a["esc_off"], a["esc_exp"])


@pytest.fixture(scope="module")
def good_arrays(uw):
    w = synthdata.student_t(256, 512, 3.0, 0.015, seed=31)
    return uw.uw_encode_host(w, uw.default_opts(chunk_syms=256)).arrays()


def test_validation_accepts_encoder_output(uw, good_arrays):
    assert uw.uw_validate_format(_buffers(uw, good_arrays).fmt) == uw.UW_OK
    # an oracle-made encoding validates too
    w = synthdata.normal(64, 256, 0.02, seed=32)
    ref = oracle.encode(w, chunk_syms=128)
    b = uw.FormatBuffers(64, 256, 12, 128, ref.lengths, ref.palette, ref.words, ref.offsets,
                         ref.sm, ref.esc_bits, ref.esc_off, ref.esc_exp)
    assert uw.uw_validate_format(b.fmt) == uw.UW_OK


def test_validation_bounds_the_stream_length(uw, good_arrays):
    """The kernels count a stream's bits (padding included) in 32 bits: a stream
    of more than 2^27 - 4 words is refused as unsupported.  (The validator does
    not read the words, so the small buffer behind the view is safe.)"""
    b = _buffers(uw, good_arrays)
    b.fmt.n_words = 2**27
    assert uw.uw_validate_format(b.fmt) == uw.UW_ERR_UNSUPPORTED
    b.fmt.n_words = 2**27 - 4
    assert uw.uw_validate_format(b.fmt) == uw.UW_OK


def _mutations(a):
    cl = a["code_len"].copy()
    nz = np.nonzero(cl)[0]
    longer = cl.copy()
    longer[nz[0]] = 13  # over the cap
    kraft = cl.copy()
    kraft[nz[:2]] = 1   # Kraft sum > 1
    off = a["chunk_off"].copy()
    off[3], off[4] = off[4], off[3]  # non-monotone
    off_end = a["chunk_off"].copy()
    off_end[-1] = a["words"].size * 32 + 1  # beyond the stream
    off_first = a["chunk_off"].copy()
    off_first[0] = 1
    pal = a["palette"].copy()
    pal[3] = pal[2]  # duplicate palette entry
    ebits = a["esc_bits"].copy()
    ebits[0] ^= 1  # escape bitmap disagrees with the group offsets
    eoff = a["esc_off"].copy()
    eoff[-1] += 1
    eexp = a["esc_exp"].copy().reshape(-1, 64)
    if eexp.shape[0]:
        eexp[0, :] = a["palette"][0]  # an escape row that needs no escaping
    words_short = a["words"][: a["words"].size - 4]
    return {
        "length over cap": dict(code_len=longer),
        "kraft > 1": dict(code_len=kraft),
        "offsets not monotone": dict(chunk_off=off),
        "offset past stream": dict(chunk_off=off_end),
        "first offset": dict(chunk_off=off_first),
        "chunk count": dict(chunk_off=a["chunk_off"][:-1]),
        "duplicate palette": dict(palette=pal),
        "escape bitmap": dict(esc_bits=ebits),
        "escape offsets": dict(esc_off=eoff),
        "escape row in palette": dict(esc_exp=eexp.reshape(-1)),
        "truncated stream": dict(words=words_short),
        "chunk size": dict(chunk_syms=100),
        "K not multiple of 64": dict(K=500),
        "cap out of range": dict(max_code_len=0),
        "no symbols": dict(code_len=np.zeros(256, np.uint8)),
    }


@pytest.mark.parametrize("name", list(_mutations({  # names only; data built per test
    "code_len": np.array([1, 1] + [0] * 254, np.uint8), "chunk_off": np.arange(6, dtype=np.uint32),
    "words": np.zeros(4, np.uint32), "palette": np.arange(16, dtype=np.uint8),
    "esc_bits": np.zeros(2, np.uint32), "esc_off": np.zeros(2, np.uint32),
    "esc_exp": np.zeros(64, np.uint8)})))
def test_validation_rejects_corruption(uw, good_arrays, name):
    assert good_arrays["esc_exp"].size > 0
    over = _mutations(good_arrays)[name]
    st = uw.uw_validate_format(_buffers(uw, good_arrays, **over).fmt)
    assert st in (uw.UW_ERR_FORMAT, uw.UW_ERR_SHAPE, uw.UW_ERR_ARG), (name, st)
