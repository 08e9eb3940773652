"""The bench's host logic on CPU.

The roofline numerators: the algorithmic bytes each kernel must move, per
weight, on weights drawn like the gate_proj workload (N(0, 0.02) BF16, about
2.6 bits per Huffman-coded exponent).

The pages' accounting: a full decode reads the stream and the sign+mantissa
bytes and writes BF16 (about 3.33 B per weight), an exponent decode writes one
byte (1.33), a transcode half a byte (0.83); the palette GEMM reads 1.5 B per
weight plus the escape rows, the BF16 and exponent GEMMs 2 B, and the
Huffman-direct product the stream and the sign+mantissa bytes (about 1.34).

The clock record: the median SM clock under load and every throttle reason
seen active during the timed region, from nvidia-smi's CSV samples.
"""
import os
import sys

import pytest

import oracle
import synthdata

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def stats():
    from tests.conftest import build_library
    build_library()
    import decode_gemm_b200 as uw
    w = synthdata.normal(1024, 4096, 0.02, seed=10)
    st = uw.uw_encode_host(w, uw.default_opts()).stats()
    return w, st


def test_stream_matches_the_oracle_code(stats):
    w, st = stats
    e = oracle.exponent_bytes(w)
    hist = oracle.exponent_histogram(e)
    lengths = oracle.package_merge_lengths(hist, 12)
    bits = int((hist * lengths.astype("int64")).sum())
    assert st["bytes_stream"] == (bits + 7) // 8
    assert st["bytes_offsets"] == (w.size // 256 + 1) * 4


@pytest.mark.parametrize("kind,lo,hi", [
    ("decode_full", 3.32, 3.35), ("decode_exp", 1.32, 1.35), ("transcode", 0.82, 0.85),
    ("decode_dot", 1.32, 1.35), ("gemm_bf16", 2.0, 2.0), ("gemm_exp", 2.0, 2.0),
    ("gemm_palette", 1.5, 1.52), ("gemv_palette", 1.5, 1.52)])
def test_algorithmic_bytes_per_weight(stats, kind, lo, hi):
    sys.path.insert(0, ROOT)
    import bench
    w, st = stats
    N, K = w.shape
    T = N * K
    b = bench._alg_bytes(kind, st, 0, N, K)  # weights alone (no tokens)
    assert lo - 1e-9 <= b / T <= hi + 1e-9, (kind, b / T)
    # X read once and Y written once on top, 2 bytes each
    M = 16
    assert bench._alg_bytes(kind, st, M, N, K) - b == (0 if kind.startswith(("decode_full",
           "decode_exp", "transcode")) else 2 * M * K + 2 * M * N)


def _sample(sm, mx=1965, reasons=("Not Active",) * 4):
    return ", ".join(["0", str(sm), str(mx), "700.00", "0x0000000000000000"] + list(reasons))


def test_clock_record():
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    cs.lines = [_sample(345), _sample(1965), _sample(1965), _sample(1950),
                _sample(1965, reasons=("Not Active", "Not Active", "Not Active", "Active")),
                "garbage line", _sample("[N/A]")]
    rec = cs.summary()
    # the idle sample before the load starts is left out of the median
    assert rec["sm_mhz"] == 1965 and rec["sm_max_mhz"] == 1965 and rec["samples"] == 5
    assert rec["reasons"] == ["sw_power_cap"]
    cs.lines = [_sample(1200, reasons=("Active", "Not Active", "Active", "Not Active"))]
    assert cs.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    cs.lines = []
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}


def test_traffic_figures_are_for_the_current_sources():
    """The DRAM traffic the bench reports beside its roofline was captured on
    the kernel sources as they are (else the bench reports none)."""
    sys.path.insert(0, ROOT)
    import bench
    fam = {"gemm_palette": "gemm", "decode_full": "decode"}
    assert set(bench.TRAFFIC) == set(fam)
    for kind, rec in bench.TRAFFIC.items():
        assert rec["src_sha"] == bench._kernel_src_sha(fam[kind]), kind
