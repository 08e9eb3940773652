"""GPU parity of the Huffman-direct product (pipeline 5) against the oracle, through the C ABI.

The kernel decodes the Huffman stream and multiplies each weight into FP32
sums without writing the weights anywhere, so two kinds of check apply:

* against the FP64 matmul (oracle.gemm_fp64) within the library's matmul
  tolerance, on row counts that leave a warp's 32 rows partly empty, chunks
  shorter than a decode round (half the lanes idle), 2 to 56 chunks per row,
  1 to 8 tokens, FP32 and BF16 outputs;
* bit-exact: with one-hot activations (X[t] = e_k) every product but one is an
  exact zero, so Y[t, n] must equal W[n, k] exactly.  Columns are chosen on
  weights whose exponent lies outside the palette (the decoder's exception
  path) and inside bursts of such weights (the exception list overflows and the
  chunk is replayed).
"""
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


def _setup(uw, w, chunk):
    import torch
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=chunk))
    need = uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, 1)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    uw.uw_set_workspace(h, ws)
    return h, ws


def _supported(uw, h, M):
    """Whether the library takes (handle, M) on pipeline 5."""
    try:
        uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, M)
        return True
    except uw.UwError as e:
        assert e.status == uw.UW_ERR_UNSUPPORTED
        return False


def _run(uw, h, x_bits, out_f32=True, **cfg):
    import torch
    M = x_bits.shape[0]
    X = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()
    Y = torch.empty((M, h.N), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    Y.fill_(float("nan"))  # poison
    uw.uw_gemm_ex(h, X, Y, M, uw.gemm_config(uw.UW_PIPE_HUFFMAN_DIRECT, **cfg), out_f32)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    return Y.float().cpu().numpy().astype(np.float64)


def _check(y, x, w, bf16_out=False):
    ref = oracle.gemm_fp64(x, w)
    ok, worst = oracle.within_tolerance(y, ref, oracle.abs_product_sum(x, w), bf16_output=bf16_out)
    assert ok, f"worst err/tol = {worst}"
    return worst


def _rare_bursts(n, k, seed, bursts=6, singles=40):
    """N(0, 0.02) weights with exponents the palette cannot hold: single ones
    (the exception list) and runs of ten in one chunk round (list overflow).
    The rare exponents (131..140: 16..8192 in magnitude) are large so that a
    missing or doubled term shows far above the tolerance."""
    w = synthdata.normal(n, k, 0.02, seed)
    rng = np.random.default_rng(seed)
    flat = w.reshape(-1)
    spots = []
    for _ in range(singles):
        p = int(rng.integers(0, flat.size))
        flat[p] = np.uint16((int(rng.integers(0, 2)) << 15) | (int(rng.integers(131, 141)) << 7)
                            | int(rng.integers(0, 128)))
        spots.append(p)
    for _ in range(bursts):
        p = int(rng.integers(0, flat.size - 10))
        for i in range(10):
            flat[p + i] = np.uint16(((i & 1) << 15) | ((131 + i) << 7) | (17 * i % 128))
            spots.append(p + i)
    return w, spots


SHAPES = [
    # (N, K, chunk_syms): chunks per row 16, 18, 56, 16, 56, 2 and 3; N not a
    # multiple of 32 except once
    (300, 1024, 64),
    (257, 1152, 64),
    (130, 3584, 64),
    (64, 4096, 256),
    (40, 14336, 256),
    (7, 128, 64),
    (45, 384, 128),
]


@pytest.mark.parametrize("N,K,chunk", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 5, 8])
def test_hdot_matches_fp64(uw, N, K, chunk, M):
    w = synthdata.student_t(N, K, 3.0, 0.015, seed=300 + N)
    x = synthdata.activations(M, K, seed=301 + K)
    h, ws = _setup(uw, w, chunk)
    assert _supported(uw, h, M)
    _check(_run(uw, h, x), x, w)
    _check(_run(uw, h, x, out_f32=False), x, w, bf16_out=True)
    h.free()


@pytest.mark.parametrize("chunk", [64, 128])
def test_hdot_exceptions_and_replay(uw, chunk):
    N, K = 96, 2048
    w, spots = _rare_bursts(N, K, seed=310 + chunk)
    x = synthdata.activations(8, K, seed=311)
    h, ws = _setup(uw, w, chunk)
    assert uw.uw_stats(h)["n_escape_rows"] > 0
    _check(_run(uw, h, x), x, w)
    # one-hot activations on the rare weights' columns: Y[t, n] = W[n, k] exactly
    cols = sorted({p % K for p in spots})
    for i in range(0, len(cols), 8):
        ks = cols[i:i + 8]
        xo = np.zeros((len(ks), K), np.uint16)
        for t, k in enumerate(ks):
            xo[t, k] = 0x3F80  # 1.0
        y = _run(uw, h, xo)
        for t, k in enumerate(ks):
            expect = oracle.to_float64(w[:, k])
            assert np.array_equal(y[t], expect), f"column {k}"
    h.free()


def test_hdot_one_hot_is_the_decoded_column(uw):
    """Every weight of a few columns (first, last, chunk and row edges) comes
    back exactly; finite corner values (+-0, subnormals) included."""
    N, K = 300, 1152
    w = synthdata.normal(N, K, 0.02, seed=320)
    w[5, 0], w[6, 1151], w[7, 64], w[8, 63] = 0x8000, 0x0001, 0x807F, 0x0080
    h, ws = _setup(uw, w, 64)
    for ks in ([0, 1, 31, 32, 63, 64, 95, 96], [127, 128, 575, 576, 1087, 1088, 1150, 1151]):
        xo = np.zeros((len(ks), K), np.uint16)
        for t, k in enumerate(ks):
            xo[t, k] = 0x3F80
        y = _run(uw, h, xo)
        for t, k in enumerate(ks):
            assert np.array_equal(y[t], oracle.to_float64(w[:, k])), f"column {k}"
    h.free()


def test_hdot_deterministic_over_grid_sizes(uw):
    """The sums are added in a fixed order: bitwise equal over repeats and
    over the number of CTAs."""
    w = synthdata.normal(500, 3584, 0.02, seed=330)
    x = synthdata.activations(3, 3584, seed=331)
    h, ws = _setup(uw, w, 64)
    ref = _run(uw, h, x)
    for ctas in (0, 0, 1, 7, 148):
        assert np.array_equal(_run(uw, h, x, gemm_ctas=ctas), ref)
    h.free()


def test_hdot_full_size(uw):
    """The 8B gate and down shapes (where a warp carries its sums over runs of
    chunk positions) at M = 1 and 8 against FP64, one-hot columns exactly, and
    bitwise equal over SM budgets."""
    for name in ("gate_14336x4096", "down_4096x14336"):
        w = synthdata.workload(name)
        K = w.shape[1]
        h, ws = _setup(uw, w, 256)
        for M in (1, 8):
            x = synthdata.activation_for(name, M)
            y = _run(uw, h, x)
            _check(y, x, w)
            if M == 1:
                for ctas in (37, 148):
                    assert np.array_equal(_run(uw, h, x, gemm_ctas=ctas), y)
        ks = [0, 255, 256, 257, 4095, K - 257, K - 256, K - 1]
        xo = np.zeros((8, K), np.uint16)
        for t, k in enumerate(ks):
            xo[t, k] = 0x3F80
        yo = _run(uw, h, xo)
        for t, k in enumerate(ks):
            assert np.array_equal(yo[t], oracle.to_float64(w[:, k])), f"{name} column {k}"
        h.free()


def test_hdot_limits_and_trace(uw):
    import torch
    w = synthdata.normal(128, 1024, 0.02, seed=340)
    h, ws = _setup(uw, w, 64)
    x = synthdata.activations(9, 1024, seed=341)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((9, 128), dtype=torch.float32, device="cuda")
    cfg = uw.gemm_config(uw.UW_PIPE_HUFFMAN_DIRECT)
    with pytest.raises(uw.UwError) as e:  # more tokens than the kernel takes
        uw.uw_gemm_ex(h, X, Y, 9, cfg, True)
    assert e.value.status == uw.UW_ERR_UNSUPPORTED
    with pytest.raises(uw.UwError) as e:
        uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, 9)
    assert e.value.status == uw.UW_ERR_UNSUPPORTED
    with pytest.raises(uw.UwError) as e:  # not a matrix-vector option
        uw.uw_gemm_ex(h, X, Y, 1, uw.gemm_config(uw.UW_PIPE_HUFFMAN_DIRECT, gemv=1), True)
    assert e.value.status == uw.UW_ERR_ARG
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    uw.uw_set_workspace(h, small)
    with pytest.raises(uw.UwError) as e:
        uw.uw_gemm_ex(h, X, Y, 1, cfg, True)
    assert e.value.status == uw.UW_ERR_WORKSPACE
    uw.uw_set_workspace(h, ws)
    uw.uw_trace_enable(h, True)
    uw.uw_gemm_ex(h, X, Y, 4, cfg, True)
    torch.cuda.synchronize()
    kinds = [k for k, _ in uw.uw_trace_read(h)]
    assert kinds == ["decode_dot"]
    uw.uw_trace_enable(h, False)
    h.free()
    # rows must be whole chunks
    for (n, k, chunk) in ((64, 1088, 128), (64, 1152, 256)):
        h = uw.uw_encode(synthdata.normal(n, k, 0.02, seed=342), uw.default_opts(chunk_syms=chunk))
        with pytest.raises(uw.UwError) as e:
            uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, 1)
        assert e.value.status == uw.UW_ERR_UNSUPPORTED
        h.free()


def test_hdot_autotune_candidate(uw):
    """At M <= 8 the autotuner weighs pipeline 5; AUTO then matches FP64
    whichever it picked, and an entry tuned at M = 1 falls back for M = 64."""
    import torch
    w = synthdata.normal(1024, 4096, 0.02, seed=350)
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=256, prepare_direct=1))
    need = max(uw.uw_workspace_bytes(h, p, 64) for p in (1, 2, 3, 4))
    ws = torch.empty(max(need, uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, 1)),
                     dtype=torch.uint8, device="cuda")
    uw.uw_set_workspace(h, ws)
    uw.uw_autotune([h], [1])
    choice = uw.uw_get_choice(h, 1)
    assert 1 <= choice["pipeline"] <= 5
    for M in (1, 64):
        x = synthdata.activations(M, 4096, seed=351 + M)
        X = torch.from_numpy(x.view(np.int16)).cuda()
        Y = torch.empty((M, 1024), dtype=torch.float32, device="cuda")
        uw.uw_gemm_f32(h, X, Y, M, uw.UW_PIPE_AUTO)
        torch.cuda.synchronize()
        assert uw.uw_last_device_status(h) == uw.UW_OK
        _check(Y.cpu().numpy().astype(np.float64), x, w)
    h.free()


def test_hdot_corrupt_stream_reports_device_status(uw):
    """Flipped stream bits (the format still valid) run through the product
    without faulting and are reported like the decoders report them; the
    process goes on to an exact product on a sound handle."""
    import torch
    N, K = 64, 1024
    w = synthdata.normal(N, K, 0.02, seed=360)
    a = uw.uw_encode_host(w, uw.default_opts(chunk_syms=64)).arrays()
    words = a["words"].copy()
    words[7] ^= 0x00F0F000
    words[90] ^= 0x12345678
    b = uw.FormatBuffers(N, K, 12, 64, a["code_len"], a["palette"], words, a["chunk_off"],
                         a["sm"], a["esc_bits"], a["esc_off"], a["esc_exp"])
    assert uw.uw_validate_format(b.fmt) == uw.UW_OK
    h = uw.uw_upload(b.fmt, uw.default_opts(chunk_syms=64, prepare_direct=0))
    ws = torch.empty(uw.uw_workspace_bytes(h, uw.UW_PIPE_HUFFMAN_DIRECT, 1), dtype=torch.uint8,
                     device="cuda")
    uw.uw_set_workspace(h, ws)
    x = synthdata.activations(2, K, seed=361)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((2, N), dtype=torch.float32, device="cuda")
    uw.uw_gemm_ex(h, X, Y, 2, uw.gemm_config(uw.UW_PIPE_HUFFMAN_DIRECT), True)
    assert uw.uw_last_device_status(h) == uw.UW_ERR_DEVICE
    h.free()
    h2, ws2 = _setup(uw, w, 64)
    _check(_run(uw, h2, x), x, w)
    h2.free()
