"""GPU parity of the preprocessing kernels (full decode, exponent-only decode,
palette transcode) against the oracle - bit-exact, through the C ABI."""
import numpy as np
import pytest

import oracle
import synthdata

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def uw():
    import torch
    assert torch.cuda.is_available()
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200
    return decode_gemm_b200


def _dev_empty(nbytes, fill=0xFF):
    import torch
    t = torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")
    t.fill_(fill)  # poison: unwritten outputs show up
    return t


def _run_all(uw, h, n, k):
    import torch
    wout = _dev_empty(2 * n * k)
    eout = _dev_empty(n * k)
    iout = _dev_empty(n * k // 2)
    uw.uw_decode_full(h, wout)
    uw.uw_decode_exp(h, eout)
    uw.uw_transcode_palette(h, iout)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    w = wout[: 2 * n * k].cpu().numpy().view(np.uint16).reshape(n, k)
    e = eout[: n * k].cpu().numpy().reshape(n, k)
    i = iout[: n * k // 2].cpu().numpy().reshape(n, k // 2)
    return w, e, i


def _expect(w, palette, esc):
    e = oracle.exponent_bytes(w)
    return e, oracle.pack_nibbles(oracle.transcode(e, palette, esc))


CASES = {
    "mat1024": lambda: (synthdata.workload("mat1024"), 1024),
    "special": lambda: (synthdata.special_values(96, 640, seed=41), 256),
    "student_t": lambda: (synthdata.student_t(300, 1280, 3.0, 0.015, seed=42), 512),
    "one_exponent": lambda: (synthdata.exponent_pattern(64, 256, [126], seed=43), 64),
    "sixteen_exponents": lambda: (synthdata.exponent_pattern(64, 512, range(112, 128), seed=44), 128),
    "all_exponents": lambda: (synthdata.exponent_pattern(64, 1024, range(256), seed=45), 1024),
    "ragged_tail": lambda: (synthdata.normal(37, 192, 0.02, seed=46), 1024),
    "many_chunks_ragged_warp": lambda: (synthdata.normal(1000, 320, 0.02, seed=47), 64),
    "big_chunks": lambda: (synthdata.normal(128, 4096, 0.02, seed=48), 4096),
    # small and mid-size chunks over special values, heavy tails, every
    # exponent, a ragged last warp and many chunk groups per warp
    "special_c64": lambda: (synthdata.special_values(96, 640, seed=52), 64),
    "student_t_c256": lambda: (synthdata.student_t(300, 1280, 3.0, 0.015, seed=53), 256),
    "all_exponents_c64": lambda: (synthdata.exponent_pattern(64, 1024, range(256), seed=54), 64),
    "ragged_c256": lambda: (synthdata.normal(1000, 320, 0.02, seed=55), 256),
    "many_groups_c256": lambda: (synthdata.normal(2048, 2048, 0.02, seed=56), 256),
}


@pytest.mark.parametrize("name", list(CASES))
def test_decode_paths_match_oracle(uw, name):
    w, chunk = CASES[name]()
    n, k = w.shape
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=chunk))
    ref = oracle.encode(w, chunk_syms=chunk) if w.size <= 1 << 20 else None
    gw, ge, gi = _run_all(uw, h, n, k)
    assert np.array_equal(gw, w)
    palette = oracle.build_palette(oracle.exponent_histogram(oracle.exponent_bytes(w)))
    esc = oracle.escape_rows(oracle.exponent_bytes(w), palette)
    e, i = _expect(w, palette, esc)
    assert np.array_equal(ge, e)
    assert np.array_equal(gi, i)
    if ref is not None:
        assert np.array_equal(palette, ref.palette)
        assert np.array_equal(oracle.transcode_from_stream(ref), gi)
    h.free()


def test_gpu_decodes_oracle_encoded_stream(uw):
    """Cross decoding: the format comes from the oracle, not the library encoder."""
    w = synthdata.student_t(200, 704, 3.0, 0.015, seed=49)
    ref = oracle.encode(w, chunk_syms=192, max_len=11)
    b = uw.FormatBuffers(200, 704, 11, 192, ref.lengths, ref.palette, ref.words, ref.offsets,
                         ref.sm, ref.esc_bits, ref.esc_off, ref.esc_exp)
    h = uw.uw_upload(b.fmt, uw.default_opts(chunk_syms=192, max_code_len=11))
    gw, ge, gi = _run_all(uw, h, 200, 704)
    assert np.array_equal(gw, w)
    assert np.array_equal(ge, oracle.decode_exp(ref))
    assert np.array_equal(gi, oracle.transcode_from_stream(ref))
    h.free()


@pytest.mark.parametrize("name", ["gate_14336x4096", "down_4096x14336"])
def test_decode_full_size_bit_exact(uw, name):
    w = synthdata.workload(name)
    n, k = w.shape
    h = uw.uw_encode(w)
    gw, ge, gi = _run_all(uw, h, n, k)
    assert np.array_equal(gw, w)
    s, e = oracle.split_fields(w)
    assert np.array_equal(ge, e)
    pal = oracle.build_palette(oracle.exponent_histogram(e))
    esc = oracle.escape_rows(e, pal)
    assert np.array_equal(gi, oracle.pack_nibbles(oracle.transcode(e, pal, esc)))
    # sampled chunks through the oracle's bit-by-bit decoder on the library stream
    a = uw.uw_encode_host(w).arrays()
    cs = int(a["chunk_syms"])
    rng = np.random.default_rng(3)
    for c in rng.choice(a["chunk_off"].size - 1, size=6, replace=False):
        syms, end = oracle.decode_chunk(a["words"], int(a["chunk_off"][c]), cs, a["code_len"])
        assert end == int(a["chunk_off"][c + 1])
        assert np.array_equal(syms, ge.reshape(-1)[c * cs:(c + 1) * cs])
    h.free()


def test_decode_heavy_tail_70b_shape(uw):
    w = synthdata.workload("gate70b_28672x8192")
    n, k = w.shape
    h = uw.uw_encode(w)
    gw, ge, gi = _run_all(uw, h, n, k)
    assert np.array_equal(gw, w)
    st = h.stats()
    assert 0.01 < st["n_escape_rows"] / st["n_rows"] < 0.1
    h.free()


def test_corrupt_stream_reports_device_status(uw):
    """A stream with flipped bits (still structurally valid) decodes without
    faulting; the kernel flags the chunks whose bit count no longer matches."""
    import torch
    w = synthdata.normal(64, 1024, 0.02, seed=50)
    a = uw.uw_encode_host(w, uw.default_opts(chunk_syms=256)).arrays()
    words = a["words"].copy()
    words[5] ^= 0x00F0F000
    words[40] ^= 0x12345678
    b = uw.FormatBuffers(64, 1024, 12, 256, a["code_len"], a["palette"], words, a["chunk_off"],
                         a["sm"], a["esc_bits"], a["esc_off"], a["esc_exp"])
    assert uw.uw_validate_format(b.fmt) == uw.UW_OK
    h = uw.uw_upload(b.fmt, uw.default_opts(chunk_syms=256, prepare_direct=0))
    out = _dev_empty(64 * 1024)
    uw.uw_decode_exp(h, out)
    assert uw.uw_last_device_status(h) == uw.UW_ERR_DEVICE
    # status is cleared by the read; a clean handle reports OK
    assert uw.uw_last_device_status(h) == uw.UW_OK
    h.free()
    torch.cuda.synchronize()


def test_device_argument_errors(uw):
    import ctypes as C
    w = synthdata.normal(16, 128, 0.02, seed=51)
    h = uw.uw_encode(w)
    assert uw.lib.uw_decode_full(h.ptr, None) == uw.UW_ERR_ARG
    t = _dev_empty(16 * 128 * 2 + 16)
    assert uw.lib.uw_decode_exp(h.ptr, C.c_void_p(t.data_ptr() + 1)) == uw.UW_ERR_ARG
    assert uw.lib.uw_decode_full(None, C.c_void_p(t.data_ptr())) == uw.UW_ERR_ARG
    h.free()


def test_bundle_load_to_device(uw, tmp_path):
    """A distribution bundle loaded straight to the device (uw_load: read,
    check, upload, load-time palette transcode) decodes bit-exactly and serves
    the direct-palette matmul within tolerance."""
    import torch
    w = synthdata.student_t(256, 512, 3.0, 0.015, seed=67)  # with escape rows
    he = uw.uw_encode_host(w, uw.default_opts(chunk_syms=128))
    path = str(tmp_path / "m.uwb")
    uw.uw_host_save(he, path)
    h = uw.uw_load(path)
    assert (h.N, h.K) == (256, 512)
    assert h.stats()["n_escape_rows"] == he.stats()["n_escape_rows"] > 0
    n, k = w.shape
    wd, ed, idx = _run_all(uw, h, n, k)
    assert np.array_equal(wd, w)
    assert np.array_equal(ed, oracle.exponent_bytes(w))
    x = synthdata.activations(8, k, seed=68)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((8, n), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(uw.uw_workspace_bytes(h, uw.UW_PIPE_PALETTE_DIRECT, 8), 256),
                     dtype=torch.uint8, device="cuda")  # split-K partial sums
    uw.uw_set_workspace(h, ws)
    uw.uw_gemm_f32(h, X, Y, 8, uw.UW_PIPE_PALETTE_DIRECT)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    ok, worst = oracle.within_tolerance(Y.cpu().numpy().astype(np.float64),
                                        oracle.gemm_fp64(x, w), oracle.abs_product_sum(x, w))
    assert ok, worst
    h.free()


# ------------------------------------------------- rows of an embedding table ----
@pytest.mark.parametrize("name,chunk", [("normal", 256), ("student_t", 128), ("special", 64),
                                        ("wide_rows", 1024)])
def test_decode_rows_bit_exact(uw, name, chunk):
    """uw_decode_rows (an embedding lookup on compressed weights): the requested
    rows, repeats and the first and last row included, bit-exact."""
    import torch
    w = {"normal": lambda: synthdata.normal(2000, 1024, 0.02, seed=180),
         "student_t": lambda: synthdata.student_t(777, 512, 3.0, 0.015, seed=181),
         "special": lambda: synthdata.special_values(300, 640, seed=182),
         "wide_rows": lambda: synthdata.normal(96, 4096, 0.02, seed=183)}[name]()
    n, k = w.shape
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=chunk, prepare_direct=0))
    rng = np.random.default_rng(184)
    for count in (1, 5, 33, 300):
        ids = rng.integers(0, n, size=count)
        ids[0] = n - 1
        if count > 1:
            ids[1] = 0
            ids[-1] = ids[0]  # a repeat
        rows = torch.from_numpy(ids.astype(np.int64)).cuda()
        out = _dev_empty(2 * count * k)
        uw.uw_decode_rows(h, rows, out)
        torch.cuda.synchronize()
        assert uw.uw_last_device_status(h) == uw.UW_OK
        got = out[: 2 * count * k].cpu().numpy().view(np.uint16).reshape(count, k)
        assert np.array_equal(got, w[ids])
    h.free()


def test_decode_rows_embedding_table_slice(uw):
    """A 32768 x 4096 slice of a vocabulary-sized embedding table: 64 token ids."""
    import torch
    w = synthdata.workload("embed_32768x4096")
    h = uw.uw_encode(w, uw.default_opts(prepare_direct=0))
    ids = np.random.default_rng(185).integers(0, w.shape[0], size=64)
    rows = torch.from_numpy(ids.astype(np.int64)).cuda()
    out = _dev_empty(2 * 64 * w.shape[1])
    uw.uw_decode_rows(h, rows, out)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    got = out[: 2 * 64 * w.shape[1]].cpu().numpy().view(np.uint16).reshape(64, -1)
    assert np.array_equal(got, w[ids])
    h.free()


def test_decode_rows_errors(uw):
    import ctypes as C
    import torch
    w = synthdata.normal(64, 320, 0.02, seed=186)  # K = 320: not a multiple of 256
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=256, prepare_direct=0))
    rows = torch.zeros(4, dtype=torch.int64, device="cuda")
    out = _dev_empty(2 * 4 * 320)
    rp, op = C.c_void_p(rows.data_ptr()), C.c_void_p(out.data_ptr())
    assert uw.lib.uw_decode_rows(h.ptr, rp, 4, op) == uw.UW_ERR_UNSUPPORTED
    h.free()
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=64, prepare_direct=0))
    assert uw.lib.uw_decode_rows(h.ptr, rp, 0, op) == uw.UW_OK
    assert uw.lib.uw_decode_rows(h.ptr, rp, -1, op) == uw.UW_ERR_SHAPE
    assert uw.lib.uw_decode_rows(h.ptr, None, 4, op) == uw.UW_ERR_ARG
    assert uw.lib.uw_decode_rows(h.ptr, C.c_void_p(rows.data_ptr() + 4), 3, op) == uw.UW_ERR_ARG
    assert uw.lib.uw_decode_rows(h.ptr, rp, 4, C.c_void_p(out.data_ptr() + 2)) == uw.UW_ERR_ARG
    # ids outside [0, N): the call returns, the device status reports it
    bad = torch.tensor([3, 64, -1, 5], dtype=torch.int64, device="cuda")
    assert uw.lib.uw_decode_rows(h.ptr, C.c_void_p(bad.data_ptr()), 4, op) == uw.UW_OK
    assert uw.uw_last_device_status(h) == uw.UW_ERR_DEVICE
    good = torch.tensor([3, 63], dtype=torch.int64, device="cuda")
    uw.uw_decode_rows(h, good, out)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    got = out[: 2 * 2 * 320].cpu().numpy().view(np.uint16).reshape(2, 320)
    assert np.array_equal(got, w[[3, 63]])
    h.free()
