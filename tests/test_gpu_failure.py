"""Failure detection without a GPU fault, through the C ABI.

A bounded wait inside the GEMM is made to run out on a flag that nothing
sets: with UW_TEST_WITHHOLD_HANDOFF in the environment the split-tile
contributors keep their ready flags back, so each tile owner's wait expires
(UW_WAIT_LIMIT_MS = 100 here).  The launch must report UW_ERR_TIMEOUT through
the device status, and the same process must go on decoding and multiplying
correctly afterwards (the kernel drained its copies and MMAs, freed its tensor
memory and returned).  The switch is read once per process, so the check runs
in a child process of its own.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import numpy as np
    import torch
    import oracle
    import synthdata
    import decode_gemm_b200 as uw

    w = synthdata.normal(1024, 1024, 0.02, seed=200)
    x = synthdata.activations(8, 1024, seed=201)
    h = uw.uw_encode(w)
    ws = torch.empty(uw.uw_workspace_bytes(h, uw.UW_PIPE_PALETTE_DIRECT, 8), dtype=torch.uint8,
                     device="cuda")
    uw.uw_set_workspace(h, ws)
    X = torch.from_numpy(x.view(np.int16)).cuda()
    Y = torch.empty((8, 1024), dtype=torch.float32, device="cuda")
    # one CTA per unit: every 128-row tile is split over 8 CTAs and every owner
    # waits for flags that never come
    uw.uw_gemm_ex(h, X, Y, 8, uw.gemm_config(uw.UW_PIPE_PALETTE_DIRECT), True)
    st = uw.uw_last_device_status(h)
    assert st == uw.UW_ERR_TIMEOUT, st
    # the status was cleared by the read
    assert uw.uw_last_device_status(h) == uw.UW_OK
    # the context still works: a decode, and a matmul with one CTA per tile (no hand-off)
    out = torch.empty(1024 * 1024, dtype=torch.int16, device="cuda")
    uw.uw_decode_full(h, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16).reshape(1024, 1024), w)
    Y.fill_(float("nan"))
    uw.uw_gemm_ex(h, X, Y, 8, uw.gemm_config(uw.UW_PIPE_PALETTE_DIRECT, gemm_ctas=8), True)
    assert uw.uw_last_device_status(h) == uw.UW_OK
    assert oracle.within_tolerance(Y.cpu().numpy().astype(np.float64), oracle.gemm_fp64(x, w),
                                   oracle.abs_product_sum(x, w))[0]
    h.free()
    print("timeout reported, context usable")
""")


def test_gemm_bounded_wait_reports_timeout():
    import torch
    assert torch.cuda.is_available()
    from tests.conftest import build_library
    build_library()
    env = dict(os.environ, UW_TEST_WITHHOLD_HANDOFF="1", UW_WAIT_LIMIT_MS="100")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "timeout reported, context usable" in r.stdout
