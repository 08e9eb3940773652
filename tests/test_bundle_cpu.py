"""Distribution bundle I/O on the host (no GPU): uw_host_save / uw_host_load.

The bundle must carry an encoding unchanged (every array byte-identical, so the
stream still equals the oracle's), and a damaged or foreign file must be refused
with a status, never accepted.
"""

import numpy as np
import pytest

import oracle
import synthdata


@pytest.fixture(scope="module")
def uw():
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200
    return decode_gemm_b200


def _arrays_equal(a, b):
    assert a.keys() == b.keys()
    for k in a:
        if isinstance(a[k], np.ndarray):
            assert np.array_equal(a[k], b[k]), k
        else:
            assert a[k] == b[k], k


@pytest.mark.parametrize("kind", ["normal", "student_t", "few_exponents"])
def test_round_trip_identical(uw, tmp_path, kind):
    if kind == "normal":
        w = synthdata.normal(300, 512, 0.02, seed=61)
    elif kind == "student_t":  # escape rows
        w = synthdata.student_t(256, 640, 3.0, 0.015, seed=62)
    else:  # at most 16 exponents: no escape rows, short code lengths
        w = synthdata.exponent_pattern(128, 256, list(range(118, 126)), seed=63)
    he = uw.uw_encode_host(w, uw.default_opts(chunk_syms=128))
    path = str(tmp_path / "m.uwb")
    uw.uw_host_save(he, path)
    back = uw.uw_host_load(path)
    _arrays_equal(he.arrays(), back.arrays())
    assert he.stats() == back.stats()  # histogram-based statistics survive the trip
    # still the oracle's encoding, byte for byte
    ref = oracle.encode(w, chunk_syms=128)
    arr = back.arrays()
    assert np.array_equal(arr["code_len"], ref.lengths)
    assert np.array_equal(arr["palette"], ref.palette)
    assert np.array_equal(arr["words"], ref.words)
    assert np.array_equal(arr["chunk_off"], ref.offsets)
    assert np.array_equal(arr["sm"], ref.sm.reshape(-1))
    assert np.array_equal(arr["esc_bits"], ref.esc_bits.reshape(-1))
    assert np.array_equal(arr["esc_off"], ref.esc_off)
    assert np.array_equal(arr["esc_exp"], ref.esc_exp.reshape(-1))


def test_file_layout(uw, tmp_path):
    """Header, sections at 16-byte offsets, 16-byte trailer (checksum, end tag)."""
    w = synthdata.normal(128, 128, 0.02, seed=64)
    he = uw.uw_encode_host(w)
    path = str(tmp_path / "m.uwb")
    uw.uw_host_save(he, path)
    raw = open(path, "rb").read()
    assert raw[:8] == b"UWBUNDLE" and raw[-8:] == b"UWBEND01"
    assert len(raw) % 16 == 0
    a = he.arrays()
    sizes = [a["words"].nbytes, a["chunk_off"].nbytes, a["sm"].nbytes, a["esc_bits"].nbytes,
             a["esc_off"].nbytes, a["esc_exp"].nbytes]
    body = 2416 + sum(s + (-s) % 16 for s in sizes)
    assert len(raw) == body + 16
    # FNV-1a 64 of the body
    h = 14695981039346656037
    for byte in raw[:body]:
        h = ((h ^ byte) * 1099511628211) & (2**64 - 1)
    assert int.from_bytes(raw[body:body + 8], "little") == h


def _saved(uw, tmp_path):
    w = synthdata.student_t(200, 320, 3.0, 0.015, seed=65)
    he = uw.uw_encode_host(w)
    path = str(tmp_path / "m.uwb")
    uw.uw_host_save(he, path)
    return path, open(path, "rb").read()


@pytest.mark.parametrize("where", ["header", "stream", "sm", "escape", "checksum", "tag"])
def test_corruption_refused(uw, tmp_path, where):
    path, raw = _saved(uw, tmp_path)
    pos = {"header": 20, "stream": 2416 + 40, "sm": len(raw) // 2, "escape": len(raw) - 40,
           "checksum": len(raw) - 12, "tag": len(raw) - 3}[where]
    bad = bytearray(raw)
    bad[pos] ^= 0x10
    open(path, "wb").write(bytes(bad))
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_load(path)
    assert e.value.status == uw.UW_ERR_FORMAT


@pytest.mark.parametrize("cut", [0, 100, 2416, -17, -1])
def test_truncated_refused(uw, tmp_path, cut):
    path, raw = _saved(uw, tmp_path)
    open(path, "wb").write(raw[:cut] if cut >= 0 else raw[:len(raw) + cut])
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_load(path)
    assert e.value.status == uw.UW_ERR_FORMAT


def test_valid_checksum_invalid_content_refused(uw, tmp_path):
    """A file whose checksum matches but whose arrays do not form an encoding
    (here: a code length above the cap) fails validation."""
    path, raw = _saved(uw, tmp_path)
    bad = bytearray(raw)
    body = len(bad) - 16
    bad[48] = 15  # code_len[8] (offset 40 + 8): longer than max_code_len 12
    h = 14695981039346656037
    for byte in bad[:body]:
        h = ((h ^ byte) * 1099511628211) & (2**64 - 1)
    bad[body:body + 8] = h.to_bytes(8, "little")
    open(path, "wb").write(bytes(bad))
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_load(path)
    assert e.value.status in (uw.UW_ERR_FORMAT, uw.UW_ERR_SHAPE)


def _rechecksum(bad):
    body = len(bad) - 16
    h = 14695981039346656037
    for byte in bad[:body]:
        h = ((h ^ byte) * 1099511628211) & (2**64 - 1)
    bad[body:body + 8] = h.to_bytes(8, "little")
    return bytes(bad)


HIST_AT = 320  # the header's int64 exponent histogram: 8 magic + 8 + 16 + 8 + 256 + 16 + 8 bytes in


@pytest.mark.parametrize("how", ["negative", "moved", "uncoded", "over"])
def test_histogram_must_match_the_matrix(uw, tmp_path, how):
    """The stored histogram only feeds the statistics, but a file whose histogram
    does not count the matrix's N*K exponents (each with a code) is refused."""
    path, raw = _saved(uw, tmp_path)
    he = uw.uw_host_load(path)
    code_len = he.arrays()["code_len"]
    hist = np.frombuffer(raw, dtype="<i8", count=256, offset=HIST_AT).copy()
    assert hist.sum() == 200 * 320 and np.all((hist > 0) <= (code_len > 0))
    a, b = [int(s) for s in np.flatnonzero(hist)[:2]]
    if how == "negative":
        hist[a], hist[b] = -1, hist[b] + hist[a] + 1      # total kept
    elif how == "moved":
        hist[a] -= 1                                       # total one short
    elif how == "uncoded":
        z = int(np.flatnonzero(code_len == 0)[0])
        hist[a] -= 1
        hist[z] += 1                                       # total kept, uncoded exponent
    else:
        hist[a] += 2**62                                   # above N*K
    bad = bytearray(raw)
    bad[HIST_AT:HIST_AT + 2048] = hist.astype("<i8").tobytes()
    open(path, "wb").write(_rechecksum(bad))
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_load(path)
    assert e.value.status == uw.UW_ERR_FORMAT


def test_io_errors(uw, tmp_path):
    w = synthdata.normal(64, 64, 0.02, seed=66)
    he = uw.uw_encode_host(w)
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_load(str(tmp_path / "missing.uwb"))
    assert e.value.status == uw.UW_ERR_IO
    with pytest.raises(uw.UwError) as e:
        uw.uw_host_save(he, str(tmp_path / "no_such_dir" / "m.uwb"))
    assert e.value.status == uw.UW_ERR_IO
    assert uw.uw_status_str(uw.UW_ERR_IO) == "file input/output failed"
