"""The bench's roofline numerators on CPU: the algorithmic bytes each kernel
must move, per weight, on weights drawn like the gate_proj workload
(N(0, 0.02) BF16, about 2.6 bits per Huffman-coded exponent).

The pages' accounting: a full decode reads the stream and the sign+mantissa
bytes and writes BF16 (about 3.33 B per weight), an exponent decode writes one
byte (1.33), a transcode half a byte (0.83); the palette GEMM reads 1.5 B per
weight plus the escape rows, the BF16 and exponent GEMMs 2 B, and the
Huffman-direct product the stream and the sign+mantissa bytes (about 1.34).
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
