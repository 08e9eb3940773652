"""GPU parity of the four pipelines' GEMM against the FP64 oracle, through the C ABI.

Acceptance: |y - y_ref| <= 1e-3 * sum_k |x w| + 1e-6 per element (FP32 output),
plus 2^-8 |y_ref| for the final rounding when the output is BF16.
P2, P3 and P4 rebuild identical BF16 tiles, so with the same variant (token
tile, CTA count) their outputs must be bitwise identical.
"""
import numpy as np
import pytest

import oracle
import synthdata

pytestmark = pytest.mark.gpu

PIPES = ["full", "exp", "palette_rt", "palette_direct"]


@pytest.fixture(scope="module")
def uw():
    import torch
    assert torch.cuda.is_available()
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200
    return decode_gemm_b200


def _upload(uw, w, chunk=1024):
    import torch
    h = uw.uw_encode(w, uw.default_opts(chunk_syms=chunk))
    return h


def _workspace(uw, h, M, pipes=PIPES, **cfg):
    import torch
    need = max(uw.uw_workspace_bytes(h, uw.PIPELINES[p], M) for p in pipes)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    uw.uw_set_workspace(h, ws)
    return ws


def _gemm(uw, h, x_bits, pipe, out_f32=True, **cfg):
    import torch
    M = x_bits.shape[0]
    X = torch.from_numpy(x_bits.view(np.int16)).cuda()
    if out_f32:
        Y = torch.empty((M, h.N), dtype=torch.float32, device="cuda")
    else:
        Y = torch.empty((M, h.N), dtype=torch.bfloat16, device="cuda")
    Y.fill_(float("nan"))  # poison
    c = uw.gemm_config(uw.PIPELINES[pipe], **cfg)
    uw.uw_gemm_ex(h, X, Y, M, c, out_f32)
    torch.cuda.synchronize()
    assert uw.uw_last_device_status(h) == uw.UW_OK
    if out_f32:
        return Y.cpu().numpy().astype(np.float64)
    return Y.float().cpu().numpy().astype(np.float64)


def _check(y, x, w, bf16_out=False):
    ref = oracle.gemm_fp64(x, w)
    bound = oracle.abs_product_sum(x, w)
    ok, worst = oracle.within_tolerance(y, ref, bound, bf16_output=bf16_out)
    assert ok, f"worst err/tol = {worst}"
    return worst


SHAPES = [
    # (M, N, K, weight maker)
    (8, 1024, 1024, "normal"),      # the 1024x1024 single-matrix case
    (1, 256, 512, "normal"),
    (17, 200, 192, "student_t"),    # ragged M, ragged N (not a multiple of 128), tiny K
    (64, 384, 640, "student_t"),
    (130, 256, 256, "normal"),      # M spans two token tiles
    (300, 128, 128, "special_finite"),
]


def _weights(kind, n, k, seed):
    if kind == "normal":
        return synthdata.normal(n, k, 0.02, seed)
    if kind == "student_t":
        return synthdata.student_t(n, k, 3.0, 0.015, seed)
    # finite corner cases: +-0 and subnormals, no Inf/NaN (they poison every sum)
    w = synthdata.normal(n, k, 0.02, seed)
    rng = np.random.default_rng(seed)
    pos = rng.choice(w.size, size=64, replace=False)
    w.reshape(-1)[pos] = np.resize(np.array([0x0000, 0x8000, 0x0001, 0x807F, 0x0080], np.uint16),
                                   64)
    return w


@pytest.mark.parametrize("M,N,K,kind", SHAPES)
@pytest.mark.parametrize("pipe", PIPES)
def test_gemm_matches_fp64(uw, M, N, K, kind, pipe):
    w = _weights(kind, N, K, seed=60 + M)
    x = synthdata.activations(M, K, seed=61 + N)
    h = _upload(uw, w, chunk=128)
    ws = _workspace(uw, h, M)
    _check(_gemm(uw, h, x, pipe), x, w)
    _check(_gemm(uw, h, x, pipe, out_f32=False), x, w, bf16_out=True)
    h.free()


def test_mat1024_public_calls(uw):
    """uw_gemm / uw_gemm_f32 with every pipeline on the 1024x1024, M=8 case."""
    import torch
    w = synthdata.workload("mat1024")
    x = synthdata.activation_for("mat1024", 8)
    h = _upload(uw, w)
    ws = _workspace(uw, h, 8)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    for p in PIPES:
        Y = torch.empty((8, 1024), dtype=torch.float32, device="cuda")
        uw.uw_gemm_f32(h, X, Y, 8, uw.PIPELINES[p])
        torch.cuda.synchronize()
        _check(Y.cpu().numpy().astype(np.float64), x, w)
        Yb = torch.empty((8, 1024), dtype=torch.bfloat16, device="cuda")
        uw.uw_gemm(h, X, Yb, 8, uw.PIPELINES[p])
        torch.cuda.synchronize()
        _check(Yb.float().cpu().numpy().astype(np.float64), x, w, bf16_out=True)
    assert uw.uw_last_device_status(h) == uw.UW_OK
    h.free()


@pytest.mark.parametrize("tile_n,ctas", [(16, 0), (32, 7), (64, 148), (128, 33)])
def test_reconstructive_pipelines_bitwise_identical(uw, tile_n, ctas):
    w = synthdata.student_t(512, 1024, 3.0, 0.015, seed=70)
    x = synthdata.activations(40, 1024, seed=71)
    h = _upload(uw, w, chunk=256)
    ws = _workspace(uw, h, 40, tile_n=tile_n)
    outs = [_gemm(uw, h, x, p, tile_n=tile_n, gemm_ctas=ctas) for p in PIPES[1:]]
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    _check(outs[0], x, w)
    h.free()


def test_escape_overflow_path(uw):
    """More than the 32 escape rows a stage stages: rows past the cap come from HBM."""
    w = synthdata.exponent_pattern(256, 512, range(90, 140), seed=72)  # ~every row escapes
    x = synthdata.activations(24, 512, seed=73)
    h = _upload(uw, w, chunk=64)
    st = h.stats()
    assert st["n_escape_rows"] > 0.9 * st["n_rows"]
    ws = _workspace(uw, h, 24)
    for p in ("palette_rt", "palette_direct"):
        _check(_gemm(uw, h, x, p), x, w)
    h.free()


@pytest.mark.parametrize("M", [1, 16, 64])
def test_gate_proj_full_size(uw, M):
    w = synthdata.workload("gate_14336x4096")
    x = synthdata.activation_for("gate_14336x4096", M)
    h = _upload(uw, w)
    ws = _workspace(uw, h, M)
    ref = oracle.gemm_fp64(x, w)
    bound = oracle.abs_product_sum(x, w)
    outs = {}
    for p in PIPES:
        y = _gemm(uw, h, x, p)
        ok, worst = oracle.within_tolerance(y, ref, bound)
        assert ok, (p, worst)
        outs[p] = y
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])
    h.free()


def _sampled_rows_check(uw, h, w, x, M, seed, n_rows):
    """Every pipeline at M tokens against FP64 on n_rows sampled token rows
    (all of them when M <= n_rows); only those rows leave the GPU.  Returns the
    sampled outputs per pipeline."""
    import torch
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(M, size=min(M, n_rows), replace=False))
    ref = oracle.gemm_fp64(x[rows], w)
    bound = oracle.abs_product_sum(x[rows], w)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((M, h.N), dtype=torch.float32, device="cuda")
    sel = torch.from_numpy(rows).cuda()
    outs = {}
    for p in PIPES:
        Y.fill_(float("nan"))
        uw.uw_gemm_ex(h, X, Y, M, uw.gemm_config(uw.PIPELINES[p]), True)
        torch.cuda.synchronize()
        assert uw.uw_last_device_status(h) == uw.UW_OK
        y = Y.index_select(0, sel).cpu().numpy().astype(np.float64)
        ok, worst = oracle.within_tolerance(y, ref, bound)
        assert ok, (p, worst)
        assert not torch.isnan(Y).any().item(), p  # every output element written
        outs[p] = y
    return outs


@pytest.fixture(scope="module")
def down8b(uw):
    """The Llama-3.1-8B down_proj shape 4096x14336, uploaded once."""
    w = synthdata.workload("down_4096x14336")
    h = _upload(uw, w)
    yield w, h
    h.free()


@pytest.mark.parametrize("M", [256, 1024, 4096])
def test_down_proj_full_size_sampled(uw, down8b, M):
    w, h = down8b
    x = synthdata.activation_for("down_4096x14336", M)
    _workspace(uw, h, M)
    outs = _sampled_rows_check(uw, h, w, x, M, seed=M, n_rows=24 if M < 4096 else 32)
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])


@pytest.fixture(scope="module")
def down70b(uw):
    """The 70B-shaped down projection 8192x28672 (Student-t weights)."""
    w = synthdata.workload("down70b_8192x28672")
    h = _upload(uw, w)
    yield w, h
    h.free()


@pytest.mark.parametrize("M", [1, 4096])
def test_down70b_shape_sampled(uw, down70b, M):
    """8192x28672 (K = 28672, the longest reduction here) with heavy tails:
    every pipeline within tolerance on sampled token rows, the reconstructive
    ones bitwise equal."""
    w, h = down70b
    assert h.stats()["n_escape_rows"] > 0
    x = synthdata.activation_for("down70b_8192x28672", M)
    _workspace(uw, h, M)
    outs = _sampled_rows_check(uw, h, w, x, M, seed=71 + M, n_rows=24)
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])


@pytest.fixture(scope="module")
def gate70b(uw):
    """The 70B-shaped gate projection (Student-t weights, many escape rows),
    uploaded once for the tests below."""
    w = synthdata.workload("gate70b_28672x8192")
    h = _upload(uw, w)
    yield w, h
    h.free()


@pytest.mark.parametrize("M", [1, 4096])
def test_gate70b_shape_sampled(uw, gate70b, M):
    """28672x8192 with heavy tails: every pipeline within tolerance on sampled
    token rows (all of them at M = 1), the reconstructive ones bitwise equal."""
    w, h = gate70b
    assert h.stats()["n_escape_rows"] > 0
    x = synthdata.activation_for("gate70b_28672x8192", M)
    _workspace(uw, h, M)
    rng = np.random.default_rng(70 + M)
    rows = np.sort(rng.choice(M, size=min(M, 24), replace=False))
    ref = oracle.gemm_fp64(x[rows], w)
    bound = oracle.abs_product_sum(x[rows], w)
    import torch
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((M, h.N), dtype=torch.float32, device="cuda")
    sel = torch.from_numpy(rows).cuda()
    outs = {}
    for p in PIPES:
        Y.fill_(float("nan"))
        uw.uw_gemm_ex(h, X, Y, M, uw.gemm_config(uw.PIPELINES[p]), True)
        torch.cuda.synchronize()
        assert uw.uw_last_device_status(h) == uw.UW_OK
        y = Y.index_select(0, sel).cpu().numpy().astype(np.float64)  # only the sampled rows leave the GPU
        ok, worst = oracle.within_tolerance(y, ref, bound)
        assert ok, (p, worst)
        outs[p] = y
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])


def test_gemm_argument_errors(uw):
    import ctypes as C
    import torch
    w = synthdata.normal(128, 256, 0.02, seed=80)
    h = uw.uw_encode(w, uw.default_opts(prepare_direct=0))
    X = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    # M == 0: nothing to do
    assert uw.lib.uw_gemm(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 0, 3) == uw.UW_OK
    # pipelines 1-3 need a workspace; none registered
    for p in (1, 2, 3):
        assert uw.lib.uw_gemm(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 4, p) \
            == uw.UW_ERR_WORKSPACE
    # pipeline 4 needs the load-time transcode, which this handle skipped
    assert uw.lib.uw_gemm(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 4, 4) \
        == uw.UW_ERR_UNSUPPORTED
    assert uw.lib.uw_gemm(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 4, 9) \
        == uw.UW_ERR_ARG
    assert uw.lib.uw_gemm(h.ptr, None, C.c_void_p(Y.data_ptr()), 4, 3) == uw.UW_ERR_ARG
    assert uw.lib.uw_gemm(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), -1, 3) \
        == uw.UW_ERR_SHAPE
    bad = uw.gemm_config(3, tile_n=24)
    assert uw.lib.uw_gemm_ex(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 4,
                             C.byref(bad), 0) == uw.UW_ERR_ARG
    h.free()


@pytest.mark.parametrize("pipe,M,tile_n", [("exp", 256, 0), ("palette_direct", 256, 0),
                                           ("full", 1, 16), ("palette_rt", 64, 32)])
def test_gemm_repeatable_bitwise(uw, pipe, M, tile_n):
    """The same call eight times gives bitwise the same Y (races show up here)."""
    w = synthdata.student_t(1024, 3584, 3.0, 0.015, seed=100 + M)
    x = synthdata.activations(M, 3584, seed=101 + M)
    h = _upload(uw, w, chunk=256)
    ws = _workspace(uw, h, M)
    first = _gemm(uw, h, x, pipe, tile_n=tile_n)
    _check(first, x, w)
    for _ in range(7):
        assert np.array_equal(_gemm(uw, h, x, pipe, tile_n=tile_n), first)
    h.free()


def test_odd_ring_depth_rejected(uw):
    import ctypes as C
    import torch
    w = synthdata.normal(128, 256, 0.02, seed=102)
    h = uw.uw_encode(w)
    X = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    for st in (1, 3, 5):
        cfg = uw.gemm_config(4, stages=st)
        assert uw.lib.uw_gemm_ex(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 4,
                                 C.byref(cfg), 0) == uw.UW_ERR_ARG
    h.free()


WIDE_SHAPES = [
    # (M, N, K, weight maker): units of 256 W rows, one 128-row half per rebuild
    # group and MMA warp
    (1, 512, 512, "normal"),
    (17, 200, 192, "student_t"),    # N < 256: the second half partly past N
    (40, 128, 256, "student_t"),    # the second half entirely past N
    (130, 640, 640, "normal"),      # two token tiles, ragged N
]


@pytest.mark.parametrize("M,N,K,kind", WIDE_SHAPES)
@pytest.mark.parametrize("pipe", PIPES)
@pytest.mark.parametrize("tile_n", [0, 256])
def test_wide_units_match_fp64(uw, M, N, K, kind, pipe, tile_n):
    """The 256-row unit shape (automatic from M = 512) on small shapes."""
    w = _weights(kind, N, K, seed=80 + M)
    x = synthdata.activations(M, K, seed=81 + N)
    h = _upload(uw, w, chunk=128)
    ws = _workspace(uw, h, M)
    for ctas in (0, 7):  # one CTA per SM, or a few so tiles split between CTAs
        y = _gemm(uw, h, x, pipe, halves=2, tile_n=tile_n, gemm_ctas=ctas)
        _check(y, x, w)
    h.free()


PAIR_SHAPES = [
    # (M, N, K, weight maker): the BF16 GEMM on CTA pairs (256 W rows x 256
    # tokens per two-SM MMA step; each CTA holds 128 rows and half the tokens)
    (256, 512, 512, "normal"),
    (300, 640, 384, "student_t"),   # ragged M: the second tile's tokens mostly past M
    (40, 200, 192, "special_finite"),  # M < 128: rank 1's token half entirely past M; N < 256
    (513, 384, 1024, "normal"),     # three token tiles, N not a multiple of 256
]


@pytest.mark.parametrize("M,N,K,kind", PAIR_SHAPES)
@pytest.mark.parametrize("out_f32", [True, False])
def test_pair_bf16_matches_fp64(uw, M, N, K, kind, out_f32):
    """Pipeline 1 with the two-SM MMA on CTA pairs, against the FP64 oracle; with
    few pairs the tiles' K ranges split between pairs (partial sums per CTA)."""
    w = _weights(kind, N, K, seed=90 + M)
    x = synthdata.activations(M, K, seed=91 + N)
    h = _upload(uw, w, chunk=128)
    ws = _workspace(uw, h, M)
    for ctas in (0, 6):  # one CTA per SM, or three pairs
        y = _gemm(uw, h, x, "full", out_f32=out_f32, pair=1, gemm_ctas=ctas)
        _check(y, x, w, bf16_out=not out_f32)
    h.free()


def test_pair_config_checked(uw):
    """CTA pairs are a BF16-GEMM variant: other pipelines and values are refused."""
    import ctypes as C
    import torch
    w = synthdata.normal(256, 256, 0.02, seed=103)
    h = uw.uw_encode(w)
    X = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    for pipe, pair, halves, want in ((4, 1, 0, uw.UW_ERR_UNSUPPORTED), (2, 1, 0, uw.UW_ERR_UNSUPPORTED),
                                     (1, 2, 0, uw.UW_ERR_ARG), (1, 1, 2, uw.UW_ERR_ARG)):
        cfg = uw.gemm_config(pipe, pair=pair, halves=halves)
        assert uw.lib.uw_gemm_ex(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 256,
                                 C.byref(cfg), 0) == want
    h.free()


PALETTE_CASES = [
    ("lookup", list(range(100, 132, 2)), 0),   # 16 exponents, not a run: palette lookup
    ("run_base0", list(range(0, 16)), 0),      # the run 0..15 (zero and subnormal weights)
    ("run_escapes", list(range(110, 126)), 40),  # a run; 40 weights get rare exponents
]


@pytest.mark.parametrize("name,exps,planted", PALETTE_CASES, ids=[c[0] for c in PALETTE_CASES])
@pytest.mark.parametrize("tile_n,halves", [(16, 1), (128, 1), (128, 2)])
def test_palette_forms_match_fp64(uw, name, exps, planted, tile_n, halves):
    """Both exponent rebuilds from indices (base + index for a palette that is
    one run, lookup otherwise), on the TMEM (tile 16) and shared-memory paths."""
    w = synthdata.exponent_pattern(384, 512, exps, seed=80 + len(exps))
    rng = np.random.default_rng(82)
    for _ in range(planted):  # exponents outside the palette: their rows escape
        r, k = int(rng.integers(0, 384)), int(rng.integers(0, 512))
        w[r, k] = (w[r, k] & 0x807F) | (int(rng.choice([90, 140])) << 7)
    h = _upload(uw, w, chunk=512)
    M = 40
    _workspace(uw, h, M)
    x = synthdata.activations(M, 512, 81)
    outs = {}
    for pipe in ("exp", "palette_rt", "palette_direct"):
        outs[pipe] = _gemm(uw, h, x, pipe, tile_n=tile_n, halves=halves)
        _check(outs[pipe], x, w)
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])
    h.free()


@pytest.mark.parametrize("pipe", PIPES)
def test_back_to_back_chain_on_one_stream(uw, pipe):
    """Launches overlap (each kernel starts its set-up before the one ahead of
    it ends and waits only before touching that kernel's data): a chain of
    GEMMs where each X is the previous Y, and preprocessing that reuses one
    workspace, enqueued with no host synchronisation, must equal the same
    calls run one at a time."""
    import torch
    K = 512
    ws_w = [synthdata.normal(K, K, 0.02, seed=120 + i) for i in range(3)]
    hs = [_upload(uw, w, chunk=256) for w in ws_w]
    M = 24
    need = max(uw.uw_workspace_bytes(h, uw.PIPELINES[pipe], M) for h in hs)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    for h in hs:
        uw.uw_set_workspace(h, ws)  # one workspace: each decode overwrites the last one's output
    x = synthdata.activations(M, K, 121)
    X0 = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)

    def chain(sync_each):
        ys = [X0]
        for h in hs:
            Y = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
            uw.uw_gemm(h, ys[-1], Y, M, uw.PIPELINES[pipe])
            if sync_each:
                torch.cuda.synchronize()
            ys.append(Y)
        torch.cuda.synchronize()
        return [y.float().cpu().numpy() for y in ys[1:]]

    ref = chain(True)
    for _ in range(3):
        got = chain(False)
        for a, b in zip(ref, got):
            assert np.array_equal(a, b)
    # and the first link against the FP64 oracle
    _check(ref[0].astype(np.float64), x, ws_w[0], bf16_out=True)
    for h in hs:
        assert uw.uw_last_device_status(h) == uw.UW_OK
        h.free()


# ---------------------------------------------------------------- M <= 2 ----
def _finite_specials(rows, cols, seed):
    """The BF16 corner cases that keep a matmul finite: +-0, subnormals, the
    smallest normal (Inf, NaN and the largest normals replaced by 1.0)."""
    w = synthdata.special_values(rows, cols, seed).copy()
    w[(w & 0x7F80) >= 0x7F00] = 0x3F80
    return w


GEMV_CASES = {
    "mat1024": lambda: synthdata.workload("mat1024"),
    "ragged_k1536": lambda: synthdata.normal(1000, 1536, 0.02, seed=170),   # a half segment
    "heavy_tail": lambda: synthdata.student_t(600, 3584, 3.0, 0.015, seed=171),
    "zeros_subnormals": lambda: _finite_specials(96, 640, seed=172),
    "not_a_run": lambda: synthdata.exponent_pattern(130, 2048, [100, 104, 108, 112, 113, 114, 115,
                                                                116, 117, 118, 119, 120, 121, 122,
                                                                126, 130, 7], seed=173),
}


@pytest.mark.parametrize("name", list(GEMV_CASES))
@pytest.mark.parametrize("M", [1, 2])
def test_gemv_matches_fp64(uw, name, M):
    """The CUDA-core matrix-vector kernel (M <= 2, uw_gemm_config.gemv = 1) of
    every pipeline against the FP64 oracle, FP32 and BF16 outputs; the
    reconstructive pipelines give bitwise the same result (same rebuilt
    weights, same summation order); escape rows, a palette that is not one run
    of exponents, a K that ends inside a 1024-weight segment."""
    w = GEMV_CASES[name]()
    x = synthdata.activations(M, w.shape[1], seed=174 + M)
    h = _upload(uw, w, chunk=256)
    _workspace(uw, h, M)
    ref = oracle.gemm_fp64(x, w)
    bound = oracle.abs_product_sum(x, w)
    outs = {}
    for p in PIPES:
        y = _gemm(uw, h, x, p, gemv=1)
        ok, worst = oracle.within_tolerance(y, ref, bound)
        assert ok, (p, worst)
        outs[p] = y
        yb = _gemm(uw, h, x, p, out_f32=False, gemv=1)
        assert oracle.within_tolerance(yb, ref, bound, bf16_output=True)[0], p
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])
    # the tensor-core GEMM (the default) agrees within tolerance
    yt = _gemm(uw, h, x, "palette_direct")
    assert oracle.within_tolerance(yt, ref, bound)[0]
    h.free()


def test_gemv_limits_and_trace(uw):
    import ctypes as C
    import torch
    w = synthdata.normal(256, 512, 0.02, seed=176)
    h = uw.uw_encode(w)
    X = torch.zeros((3, 512), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((3, 256), dtype=torch.float32, device="cuda")
    c = uw.gemm_config(4, gemv=1)
    assert uw.lib.uw_gemm_ex(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 3,
                             C.byref(c), 1) == uw.UW_ERR_UNSUPPORTED
    for bad in (2, -1):
        c = uw.gemm_config(4, gemv=bad)
        assert uw.lib.uw_gemm_ex(h.ptr, C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr()), 1,
                                 C.byref(c), 1) == uw.UW_ERR_ARG
    # pipeline 4 at M = 1 needs no workspace on this path; traced as the matrix-vector kernel
    uw.uw_trace_enable(h, True)
    uw.uw_gemm_ex(h, X, Y, 1, uw.gemm_config(4, gemv=1), True)
    kinds = [k for k, _ in uw.uw_trace_read(h)]
    assert kinds == ["gemv_palette"]
    assert uw.uw_last_device_status(h) == uw.UW_OK
    h.free()


@pytest.mark.parametrize("name,M", [("gate_14336x4096", 1), ("down70b_8192x28672", 2)])
def test_gemv_full_size(uw, name, M):
    """Full-size shapes on the matrix-vector kernel: every output row against
    FP64 (gate, M = 1) and the 70B down shape (K = 28672, 28 segments)."""
    w = synthdata.workload(name)
    x = synthdata.activation_for(name, M)
    h = _upload(uw, w, chunk=256)
    _workspace(uw, h, M)
    ref = oracle.gemm_fp64(x, w)
    bound = oracle.abs_product_sum(x, w)
    for p in PIPES:
        y = _gemm(uw, h, x, p, gemv=1)
        ok, worst = oracle.within_tolerance(y, ref, bound)
        assert ok, (p, worst)
    h.free()


# ------------------------------------------------- attention-shaped weights ----
@pytest.mark.parametrize("name", ["attn_q_4096x4096", "attn_kv_1024x4096"])
@pytest.mark.parametrize("M", [1, 64, 1024])
def test_attention_projections(uw, name, M):
    """The format on Llama-3.1-8B attention projections (q/o 4096x4096, k/v
    1024x4096): every pipeline against FP64 (sampled token rows at M = 1024),
    the reconstructive ones bitwise equal."""
    w = synthdata.workload(name)
    x = synthdata.activation_for(name, M)
    h = _upload(uw, w, chunk=256)
    _workspace(uw, h, M)
    outs = _sampled_rows_check(uw, h, w, x, M, seed=190 + M, n_rows=M if M <= 64 else 24)
    assert np.array_equal(outs["exp"], outs["palette_rt"])
    assert np.array_equal(outs["exp"], outs["palette_direct"])
    h.free()
