"""The matmul that consumes the weights (oracle; test infrastructure only).

*Unweight*, section "How the reconstructive matmul works": the reconstructed
BF16 weights feed the tensor cores directly; the output is the ordinary linear
layer ``Y = X W^T`` (PyTorch ``Linear`` layout, W is [N, K]).  Because the
compression is lossless, the exact result has a plain definition:

    y[m, n] = sum_k x[m, k] * w[n, k]        (computed in float64)

Acceptance (the tolerance fixed for this build): an FP32-accumulated result
``y`` passes when ``|y - y_ref| <= 1e-3 * sum_k |x[m,k] * w[n,k]| + 1e-6`` for
every element.  Reading taken for BF16 outputs: the result is additionally
rounded once to BF16, so ``2**-8 * |y_ref|`` (half an ulp of BF16 relative, a
full ulp to be safe with round-to-nearest-even ties) is added to the bound.
"""
from __future__ import annotations

import math

import numpy as np

from .bf16 import to_float64


def gemm_fp64(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """y = x w^T in float64 from raw BF16 bits (x [M, K], w [N, K])."""
    return to_float64(x_bits) @ to_float64(w_bits).T


def abs_product_sum(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """sum_k |x[m,k] * w[n,k]| in float64."""
    return np.abs(to_float64(x_bits)) @ np.abs(to_float64(w_bits)).T


def gemm_entry_fsum(x_bits: np.ndarray, w_bits: np.ndarray, m: int, n: int) -> float:
    """One output element summed exactly (math.fsum) - for sampled checks."""
    x = to_float64(np.asarray(x_bits)[m])
    w = to_float64(np.asarray(w_bits)[n])
    return math.fsum((x * w).tolist())


def swiglu(g_bits: np.ndarray, u_bits: np.ndarray) -> np.ndarray:
    """SwiGLU of the MLP block between the gate/up and the down projection:
    ``h = SiLU(g) * u`` with ``SiLU(g) = g / (1 + exp(-g))``, from BF16 inputs,
    in float64 (*Unweight*, results section: the method targets SwiGLU MLPs).
    Reading taken: the GPU computes it in FP32 and rounds h once to BF16, so a
    result within one BF16 rounding (2**-8 relative) of this value is exact."""
    g = to_float64(g_bits)
    u = to_float64(u_bits)
    return g / (1.0 + np.exp(-g)) * u


def tolerance(bound: np.ndarray, y_ref: np.ndarray, bf16_output: bool) -> np.ndarray:
    tol = 1e-3 * bound + 1e-6
    if bf16_output:
        tol = tol + 2.0 ** -8 * np.abs(y_ref)
    return tol


def within_tolerance(y: np.ndarray, y_ref: np.ndarray, bound: np.ndarray,
                     bf16_output: bool = False):
    """(ok, worst ratio |err|/tol) for the acceptance rule above."""
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - y_ref)
    tol = tolerance(bound, y_ref, bf16_output)
    if not np.all(np.isfinite(y)):
        return False, float("inf")
    ratio = float((err / tol).max()) if err.size else 0.0
    return bool(np.all(err <= tol)), ratio
