"""The bench's multi-rank logic on CPU (gloo, world size 2): replicas only, the
job's time is the slowest rank's, the whole-job rate counts every rank's bytes;
the reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [12.5, 20.0][rank]            # the ranks' device times (ms)
        ms = bench.max_over_ranks(mine, world, device="cpu")
        rate = bench.job_rate(3.0e9, ms, world)  # 3 GB per rank in the timed region
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got = json.load(open(tmp_path / f"r{r}.json"))
        assert got["ms"] == 20.0                      # every rank sees the slowest time
        assert got["rate"] == pytest.approx(2 * 3.0e9 / 20e-3 / 1e9)  # 300 GB/s for the job


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_rate(1e9, 1.0, 1) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun the reference arm (the oracle on the host) runs on rank 0
    only; every other rank exits 0 without printing."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_reference_arm_rank0_line():
    """Rank 0 of the reference arm prints one JSON line: the oracle timed on a
    bounded sample, with the contract's keys."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_source_digest_ignores_comments_only():
    """The traffic figures stay valid across comment and layout edits, not code edits."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) {  // doubles x\n  return 2 * x; /* twice */\n}\n"
    b = "// header\nint f(int x) {\n\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert len(bench._kernel_src_sha("gemm")) == 16 and bench._kernel_src_sha("decode") != bench._kernel_src_sha("gemm")
