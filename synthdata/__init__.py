"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module only draws random numbers and rounds them to BF16.  It holds none of
the compression method's arithmetic (no field split, no coding, no palette), so
that the CPU oracle and the CUDA path can both take their inputs from here while
sharing no code with one another.

Every matrix is returned as raw BF16 bit patterns in a ``numpy.uint16`` array,
row-major, shaped like ``torch.nn.Linear.weight`` (``[N, K]`` for weights,
``[M, K]`` for activations).

Workloads (the weights the method is measured on are Llama-3.1-8B MLP
projections, which are not available here; these draws stand in for them):

* ``normal``: ``torch.randn(float32) * std`` rounded to BF16 (round to nearest
  even), drawn with ``torch.Generator('cpu').manual_seed(seed)``.
* ``student_t``: ``numpy.random.default_rng(seed).standard_t(nu) * std /
  sqrt(nu / (nu - 2))`` (unit-variance Student-t scaled to ``std``), rounded to
  BF16 through torch.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "to_bf16_bits", "bf16_bits_to_float", "normal", "student_t", "activations",
    "special_values", "exponent_pattern", "WORKLOADS", "workload",
]


def to_bf16_bits(a) -> np.ndarray:
    """Round a float array to BF16 (round to nearest even) and return its bits."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Widen raw BF16 bits to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal(rows: int, cols: int, std: float, seed: int) -> np.ndarray:
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn((rows, cols), generator=g, dtype=torch.float32) * float(std)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def student_t(rows: int, cols: int, nu: float, std: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(int(seed))
    x = rng.standard_t(nu, size=(rows, cols)) * (std / np.sqrt(nu / (nu - 2.0)))
    return to_bf16_bits(x.astype(np.float32))


def activations(m: int, k: int, seed: int) -> np.ndarray:
    """X ~ N(0, 1) in BF16."""
    return normal(m, k, 1.0, seed)


def special_values(rows: int, cols: int, seed: int) -> np.ndarray:
    """A weight matrix salted with every BF16 corner case.

    Mostly N(0, 0.02) draws, with +-0, subnormals (exponent byte 0), +-Inf and
    NaN payloads (exponent byte 255) and very large / very small normals planted
    at seeded positions.  Used for the lossless round-trip edge cases.
    """
    w = normal(rows, cols, 0.02, seed).copy()
    rng = np.random.default_rng(int(seed) + 7)
    flat = w.reshape(-1)
    n = flat.size
    specials = np.array(
        [0x0000, 0x8000,            # +0, -0
         0x0001, 0x8001, 0x007F,    # subnormals
         0x7F80, 0xFF80,            # +-Inf
         0x7FC0, 0xFFC1, 0x7F81,    # NaN payloads
         0x7F7F, 0x0080, 0x3F80],   # max normal, min normal, 1.0
        dtype=np.uint16)
    pos = rng.choice(n, size=min(n, 4 * specials.size), replace=False)
    flat[pos] = np.resize(specials, pos.size)
    return w


def exponent_pattern(rows: int, cols: int, exponents, seed: int) -> np.ndarray:
    """Weights whose exponent bytes are drawn uniformly from ``exponents``.

    Sign and mantissa bits are uniform random.  Used to build degenerate
    alphabets (one distinct exponent, exactly 16, more than 16 ...).
    """
    rng = np.random.default_rng(int(seed))
    exps = np.asarray(list(exponents), dtype=np.uint16)
    e = exps[rng.integers(0, exps.size, size=(rows, cols))]
    sign = rng.integers(0, 2, size=(rows, cols), dtype=np.uint16)
    mant = rng.integers(0, 128, size=(rows, cols), dtype=np.uint16)
    return ((sign << 15) | (e << 7) | mant).astype(np.uint16)


# name -> (N, K, kind, std, seed_w, seed_x_base, Ms)
WORKLOADS = {
    # single 1024x1024 matrix, X 8x1024
    "mat1024": dict(N=1024, K=1024, kind="normal", std=0.02, seed_w=0, seed_x=1, Ms=(8,)),
    # Llama-3.1-8B gate_proj shape
    "gate_14336x4096": dict(N=14336, K=4096, kind="normal", std=0.02, seed_w=10, seed_x=11,
                            Ms=(1, 16, 64)),
    # Llama-3.1-8B down_proj shape
    "down_4096x14336": dict(N=4096, K=14336, kind="normal", std=0.014, seed_w=20, seed_x=21,
                            Ms=(256, 1024, 4096)),
    # 70B-shaped projections with heavy tails
    "gate70b_28672x8192": dict(N=28672, K=8192, kind="student_t", std=0.015, nu=3.0, seed_w=50,
                               seed_x=52, Ms=(1, 4096)),
    "down70b_8192x28672": dict(N=8192, K=28672, kind="student_t", std=0.015, nu=3.0, seed_w=51,
                               seed_x=53, Ms=(1, 4096)),
    # Llama-3.1-8B attention projections (q/o 4096x4096, k/v 1024x4096 with
    # grouped-query attention) and a vocabulary-sized embedding table
    # (128256 x 4096 in the model; a 32768-row slice here), N(0, 0.02)
    "attn_q_4096x4096": dict(N=4096, K=4096, kind="normal", std=0.02, seed_w=60, seed_x=61,
                             Ms=(1, 64, 1024)),
    "attn_kv_1024x4096": dict(N=1024, K=4096, kind="normal", std=0.02, seed_w=62, seed_x=63,
                              Ms=(1, 64, 1024)),
    "embed_32768x4096": dict(N=32768, K=4096, kind="normal", std=0.02, seed_w=64, seed_x=65,
                             Ms=(1, 64)),
}


def workload(name: str, rows: int | None = None):
    """Weights of a named workload (optionally only the first ``rows`` rows).

    For the normal workloads a prefix of rows equals the first rows of the
    full draw (torch fills row-major from one stream; a test checks this), so
    small-case checks see the same numbers as the full matrix.
    """
    w = WORKLOADS[name]
    n = w["N"] if rows is None else int(rows)
    if w["kind"] == "normal":
        return normal(n, w["K"], w["std"], w["seed_w"])
    return student_t(n, w["K"], w["nu"], w["std"], w["seed_w"])


def activation_for(name: str, m: int) -> np.ndarray:
    w = WORKLOADS[name]
    return activations(m, w["K"], w["seed_x"] + m)
