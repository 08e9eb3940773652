"""MLP stack driver, SwiGLU, autotuner and profile I/O on the GPU, through the C ABI.

Every projection of the stacked forward is checked against the FP64 oracle
given the GPU's own BF16 input to it (uw_mlp_forward_record), with and without
the side-stream overlap and the decoder/GEMM SM split.  The stacked forward
must also equal, bit for bit, the same projections run one by one through
uw_gemm_ex with the same variants plus uw_swiglu (the split only changes which
SMs run what, not the arithmetic, when the GEMM CTA count is the same).
"""
import json
import os
import tempfile

import numpy as np
import pytest

import oracle
import synthdata

pytestmark = pytest.mark.gpu

D, F = 256, 768


@pytest.fixture(scope="module")
def uw():
    import torch
    assert torch.cuda.is_available()
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200
    return decode_gemm_b200


def test_swiglu_matches_oracle(uw):
    import torch
    n = 3 * 1024 + 5  # vector body plus a scalar tail
    g = synthdata.normal(1, n, 2.0, seed=110).reshape(-1)
    u = synthdata.normal(1, n, 1.0, seed=111).reshape(-1)
    G = torch.from_numpy(g.view(np.int16)).cuda()
    U = torch.from_numpy(u.view(np.int16)).cuda()
    Hd = torch.empty_like(G)
    uw.uw_swiglu(G, U, Hd)
    torch.cuda.synchronize()
    h = oracle.to_float64(Hd.cpu().numpy().view(np.uint16))
    ref = oracle.swiglu(g, u)
    assert np.all(np.abs(h - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)


def _layers(uw, n_layers, pipes):
    """Handles for n_layers blocks; pipes[l] = (gate, up, down) pipelines."""
    layers, weights = [], []
    for l in range(n_layers):
        wg = synthdata.normal(F, D, 0.05, seed=120 + 3 * l)
        wu = synthdata.normal(F, D, 0.05, seed=121 + 3 * l)
        wd = synthdata.student_t(D, F, 3.0, 0.03, seed=122 + 3 * l)
        hs = tuple(uw.uw_encode(w, uw.default_opts(chunk_syms=128)) for w in (wg, wu, wd))
        layers.append(hs)
        weights.append((wg, wu, wd))
    return layers, weights


def _load_pipelines(uw, layers, pipes, M, gemm_ctas=0, gemv=0):
    """Pin each projection's pipeline (and matmul kernel) for M through a profile file."""
    flat = [h for trio in layers for h in trio]
    prof = {"version": 1, "handles": []}
    for (trio, ps) in zip(layers, pipes):
        for h, p in zip(trio, ps):
            prof["handles"].append({"N": h.N, "K": h.K, "choices": [
                {"M": M, "pipeline": p, "tile_n": 0, "stages": 0, "gemm_ctas": gemm_ctas,
                 "decode_ctas": 0, "gemv": gemv}]})
    with tempfile.NamedTemporaryFile("w", suffix=".json", delete=False) as f:
        json.dump(prof, f)
        path = f.name
    uw.uw_load_profile(flat, path)
    os.unlink(path)


def _reference(uw, layers, x, M, gemm_ctas=0):
    """The block, one public call at a time."""
    import torch
    cur = torch.from_numpy(x.view(np.int16)).cuda()
    for trio in layers:
        outs = []
        for h in trio[:2]:
            c = uw.uw_get_choice(h, M)
            cfg = uw.gemm_config(c["pipeline"], c["tile_n"], c["stages"], c["gemm_ctas"] or gemm_ctas)
            Y = torch.empty((M, F), dtype=torch.int16, device="cuda")
            uw.uw_gemm_ex(h, cur, Y, M, cfg, False)
            outs.append(Y)
        H = torch.empty_like(outs[0])
        uw.uw_swiglu(outs[0], outs[1], H)
        c = uw.uw_get_choice(trio[2], M)
        cfg = uw.gemm_config(c["pipeline"], c["tile_n"], c["stages"], c["gemm_ctas"] or gemm_ctas)
        nxt = torch.empty((M, D), dtype=torch.int16, device="cuda")
        uw.uw_gemm_ex(trio[2], H, nxt, M, cfg, False)
        cur = nxt
    torch.cuda.synchronize()
    return cur.cpu().numpy()


PIPES = [(1, 4, 2), (3, 2, 4), (4, 4, 4)]  # hard and easy projections mixed


@pytest.mark.parametrize("M", [1, 24])
def test_mlp_forward_equals_call_sequence(uw, M):
    import torch
    layers, weights = _layers(uw, 3, PIPES)
    _load_pipelines(uw, layers, PIPES, M)
    flat = [h for trio in layers for h in trio]
    for h in flat:  # workspaces for the call-by-call reference
        ws = torch.empty(max(uw.uw_workspace_bytes(h, p, M) for p in (1, 2, 3, 4)),
                         dtype=torch.uint8, device="cuda")
        uw.uw_set_workspace(h, ws)
    x = synthdata.activations(M, D, seed=130 + M)
    ref = _reference(uw, layers, x, M)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    side = torch.cuda.Stream()
    for opts in (uw.mlp_opts(False), uw.mlp_opts(True), uw.mlp_opts(True, decode_ctas=4)):
        need = uw.uw_mlp_workspace_bytes(layers, M, opts)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        Y = torch.full((M, D), -1, dtype=torch.int16, device="cuda")
        uw.uw_mlp_forward(layers, X, Y, M, ws, opts, side_stream=side)
        torch.cuda.synchronize()
        assert np.array_equal(Y.cpu().numpy(), ref), opts.as_dict()
    for h in flat:
        assert uw.uw_last_device_status(h) == uw.UW_OK
    # first layer's gate against the FP64 oracle (the GEMMs are checked in depth elsewhere)
    Yg = torch.empty((M, F), dtype=torch.float32, device="cuda")
    uw.uw_gemm_f32(layers[0][0], X, Yg, M, uw.UW_PIPE_AUTO)
    torch.cuda.synchronize()
    assert oracle.within_tolerance(Yg.cpu().numpy().astype(np.float64),
                                   oracle.gemm_fp64(x, weights[0][0]),
                                   oracle.abs_product_sum(x, weights[0][0]))[0]
    for h in flat:
        h.free()


SPLITS = {
    "serial": dict(overlap=False),
    "overlap": dict(overlap=True),
    "overlap_decode4": dict(overlap=True, decode_ctas=4),
    "overlap_decode4_gemm100": dict(overlap=True, decode_ctas=4, gemm_ctas=100),
    "serial_gemm60": dict(overlap=False, gemm_ctas=60),
    "overlap_matvec": dict(overlap=True),  # every projection on the matrix-vector kernel
    "overlap_hdot": dict(overlap=True),  # pipeline 5 mixed in (HDOT_PIPES)
}
# the Huffman-direct product (pipeline 5, no preprocessing) among hard and easy projections
HDOT_PIPES = [(5, 4, 2), (3, 5, 5), (5, 5, 4)]


@pytest.mark.parametrize("M", [1, 2, 24])
@pytest.mark.parametrize("split", list(SPLITS))
def test_mlp_stack_projections_against_fp64(uw, M, split):
    """Every projection of a 3-layer stack run by uw_mlp_forward (hard and easy
    pipelines mixed; preprocessing overlap and SM split on and off) against the
    FP64 oracle, each given the GPU's own BF16 input to it; SwiGLU against the
    oracle given the GPU's own g and u (*Unweight*, "Sharing the GPU between
    decode and compute")."""
    import torch
    gemv = 1 if split == "overlap_matvec" else 0
    if gemv and M > 2:
        pytest.skip("the matrix-vector kernel serves M <= 2")
    pipes = HDOT_PIPES if split == "overlap_hdot" else PIPES
    layers, weights = _layers(uw, 3, pipes)
    _load_pipelines(uw, layers, pipes, M, gemv=gemv)
    x = synthdata.activations(M, D, seed=160 + M)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    side = torch.cuda.Stream()
    opts = uw.mlp_opts(**SPLITS[split])
    ws = torch.empty(uw.uw_mlp_workspace_bytes(layers, M, opts), dtype=torch.uint8, device="cuda")
    per = M * (3 * F + D)
    act = torch.full((len(layers) * per,), -1, dtype=torch.int16, device="cuda")
    Y = torch.full((M, D), -1, dtype=torch.int16, device="cuda")
    uw.uw_mlp_forward_record(layers, X, Y, M, ws, act, opts, side_stream=side)
    torch.cuda.synchronize()
    a = act.cpu().numpy().view(np.uint16).reshape(len(layers), per)
    cur = x
    for l, (wg, wu, wd) in enumerate(weights):
        g = a[l, :M * F].reshape(M, F)
        u = a[l, M * F:2 * M * F].reshape(M, F)
        hh = a[l, 2 * M * F:3 * M * F].reshape(M, F)
        nxt = a[l, 3 * M * F:].reshape(M, D)
        for name, out, inp, w in (("gate", g, cur, wg), ("up", u, cur, wu), ("down", nxt, hh, wd)):
            ok, worst = oracle.within_tolerance(oracle.to_float64(out), oracle.gemm_fp64(inp, w),
                                                oracle.abs_product_sum(inp, w), bf16_output=True)
            assert ok, (split, l, name, pipes[l], worst)
        ref = oracle.swiglu(g, u)
        assert np.all(np.abs(oracle.to_float64(hh) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
        cur = nxt
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), cur)
    # recording changes nothing: the plain forward gives the same Y bit for bit
    Y2 = torch.full((M, D), -1, dtype=torch.int16, device="cuda")
    uw.uw_mlp_forward(layers, X, Y2, M, ws, opts, side_stream=side)
    torch.cuda.synchronize()
    assert np.array_equal(Y2.cpu().numpy().view(np.uint16), cur)
    for trio in layers:
        for h in trio:
            assert uw.uw_last_device_status(h) == uw.UW_OK
            h.free()


def test_mlp_split_tuner_and_gemm_cta_cap(uw):
    import torch
    M = 8
    layers, _ = _layers(uw, 2, PIPES[:2])
    _load_pipelines(uw, layers, PIPES[:2], M)
    x = synthdata.activations(M, D, seed=140)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    side = torch.cuda.Stream()
    opts = uw.mlp_opts(True, decode_ctas=8, gemm_ctas=100)
    ws = torch.empty(uw.uw_mlp_workspace_bytes(layers, M, opts), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    best = uw.uw_mlp_tune_split(layers, X, Y, M, ws, side_stream=side)
    assert best.overlap == 1 and best.decode_ctas >= 0 and best.gemm_ctas >= 0
    # a GEMM CTA cap gives the same result as the call sequence with that cap
    flat = [h for trio in layers for h in trio]
    for h in flat:
        wsh = torch.empty(max(uw.uw_workspace_bytes(h, p, M) for p in (1, 2, 3, 4)),
                          dtype=torch.uint8, device="cuda")
        uw.uw_set_workspace(h, wsh)
    ref = _reference(uw, layers, x, M, gemm_ctas=100)
    uw.uw_mlp_forward(layers, X, Y, M, ws, opts, side_stream=side)
    torch.cuda.synchronize()
    assert np.array_equal(Y.cpu().numpy(), ref)
    for h in flat:
        h.free()


def test_autotune_profile_roundtrip(uw, tmp_path):
    import torch
    wg = synthdata.normal(1024, 512, 0.02, seed=150)
    wd = synthdata.normal(512, 1024, 0.02, seed=151)
    hs = [uw.uw_encode(w) for w in (wg, wd)]
    for h in hs:
        ws = torch.empty(max(uw.uw_workspace_bytes(h, p, 64) for p in (1, 2, 3, 4)),
                         dtype=torch.uint8, device="cuda")
        uw.uw_set_workspace(h, ws)
        h._keep = ws
    path = str(tmp_path / "profile.json")
    uw.uw_autotune(hs, [1, 64], path)
    prof = json.load(open(path))
    assert [(e["N"], e["K"]) for e in prof["handles"]] == [(1024, 512), (512, 1024)]
    for e in prof["handles"]:
        assert [c["M"] for c in e["choices"]] == [1, 64]
        for c in e["choices"]:
            assert 1 <= c["pipeline"] <= 4 and c["us"] > 0
    chosen = [[uw.uw_get_choice(h, m) for m in (1, 64)] for h in hs]
    # fresh handles pick the same variants after loading the file
    hs2 = [uw.uw_encode(w) for w in (wg, wd)]
    uw.uw_load_profile(hs2, path)
    assert [[uw.uw_get_choice(h, m) for m in (1, 64)] for h in hs2] == chosen
    # the tuned (AUTO) matmul is still correct
    for h, w in zip(hs, (wg, wd)):
        for M in (1, 64):
            x = synthdata.activations(M, w.shape[1], seed=152 + M)
            Y = torch.empty((M, w.shape[0]), dtype=torch.float32, device="cuda")
            uw.uw_gemm_f32(h, torch.from_numpy(x.view(np.int16)).cuda(), Y, M, uw.UW_PIPE_AUTO)
            torch.cuda.synchronize()
            assert oracle.within_tolerance(Y.cpu().numpy().astype(np.float64),
                                           oracle.gemm_fp64(x, w), oracle.abs_product_sum(x, w))[0]
    # malformed or mismatched profiles are rejected and leave the handles alone
    bad = tmp_path / "bad.json"
    bad.write_text('{"version": 1, "handles": [{"N": 1, "K": 512, "choices": []}, '
                   '{"N": 512, "K": 1024, "choices": []}]}')
    with pytest.raises(uw.UwError):
        uw.uw_load_profile(hs2, str(bad))
    bad.write_text("{not json")
    with pytest.raises(uw.UwError):
        uw.uw_load_profile(hs2, str(bad))
    assert [[uw.uw_get_choice(h, m) for m in (1, 64)] for h in hs2] == chosen
    for h in hs + hs2:
        h.free()
