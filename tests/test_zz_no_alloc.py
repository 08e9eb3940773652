"""The allocation-free matmul (uw_gemm_palette_noalloc) against uw_gemm.

For callers that cannot allocate device memory while they run (a locked or
fully planned allocator): the split-K scratch lives in a fixed array inside
the library.  This file is collected last so that, should it fail, a run that
stops at the first failure has already run every other test; it also passes
on its own in a fresh process.
"""
import ctypes as C

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


@pytest.mark.parametrize("N,K,M,kind", [(1024, 1024, 8, "normal"), (2048, 4096, 1, "normal"),
                                        (640, 1536, 64, "student_t"), (200, 512, 17, "student_t")])
def test_noalloc_matches_uw_gemm_twice(uw, N, K, M, kind):
    import torch
    if kind == "normal":
        w = synthdata.normal(N, K, 0.02, seed=90 + M)
    else:
        w = synthdata.student_t(N, K, 3.0, 0.015, seed=90 + M)
    x = synthdata.activations(M, K, seed=91 + M)
    h = uw.uw_encode(w)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    # the existing entry point, with a registered workspace
    ws = torch.empty(uw.uw_workspace_bytes(h, uw.UW_PIPE_PALETTE_DIRECT, M), dtype=torch.uint8,
                     device="cuda")
    uw.uw_set_workspace(h, ws)
    ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
    uw.uw_gemm_f32(h, X, ref, M, uw.UW_PIPE_PALETTE_DIRECT)
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy().astype(np.float64)
    y_exact = oracle.gemm_fp64(x, w)
    bound = oracle.abs_product_sum(x, w)
    assert oracle.within_tolerance(ref_np, y_exact, bound)[0]
    # the allocation-free call, twice in a row, through the C ABI; the output
    # buffers are made before the calls, so device memory use around each call
    # shows what the call itself allocated
    outs = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
            for _ in range(2)]
    torch.cuda.synchronize()
    for Y in outs:
        free_before, _ = torch.cuda.mem_get_info()
        torch_before = torch.cuda.memory_allocated()
        st = uw.lib.uw_gemm_palette_noalloc(h.ptr, C.c_void_p(X.data_ptr()),
                                            C.c_void_p(Y.data_ptr()), M, 1)
        assert st == uw.UW_OK, uw.uw_status_str(st)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.cuda.memory_allocated() == torch_before
        y = Y.cpu().numpy().astype(np.float64)
        ok, worst = oracle.within_tolerance(y, ref_np, bound)
        assert ok, worst
        assert oracle.within_tolerance(y, y_exact, bound)[0]
    # BF16 output as well
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert uw.lib.uw_gemm_palette_noalloc(h.ptr, C.c_void_p(X.data_ptr()),
                                          C.c_void_p(Yb.data_ptr()), M, 0) == uw.UW_OK
    torch.cuda.synchronize()
    assert oracle.within_tolerance(Yb.float().cpu().numpy().astype(np.float64), y_exact, bound,
                                   bf16_output=True)[0]
    assert uw.uw_last_device_status(h) == uw.UW_OK
    h.free()


def test_noalloc_rejects_what_it_cannot_hold(uw):
    import torch
    w = synthdata.normal(256, 512, 0.02, seed=95)
    h = uw.uw_encode(w)
    X = torch.zeros((65, 512), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((65, 256), dtype=torch.float32, device="cuda")
    xp, yp = C.c_void_p(X.data_ptr()), C.c_void_p(Y.data_ptr())
    assert uw.lib.uw_gemm_palette_noalloc(h.ptr, xp, yp, 65, 1) == uw.UW_ERR_SHAPE
    assert uw.lib.uw_gemm_palette_noalloc(h.ptr, xp, yp, 0, 1) == uw.UW_OK
    assert uw.lib.uw_gemm_palette_noalloc(None, xp, yp, 4, 1) == uw.UW_ERR_ARG
    h.free()
    h2 = uw.uw_encode(w, uw.default_opts(prepare_direct=0))
    assert uw.lib.uw_gemm_palette_noalloc(h2.ptr, xp, yp, 4, 1) == uw.UW_ERR_UNSUPPORTED
    h2.free()
