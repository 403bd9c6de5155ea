"""The SwiGLU epilogue's reciprocal (the fc1 epilogue computes
silu(g) = g / (1 + e^-g) with a bit-level seed of 1/d refined by three
Newton-Raphson steps): the seed constant's error over a binade and the fp32
result after the three steps, checked on the host over every mantissa of
[1, 2) (the error pattern repeats in every binade of d >= 1)."""

import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "mixture_experts_layer_grouped_b200", "csrc", "grouped_gemm.cuh")


def _seed_constant():
    m = re.search(r"constexpr int kRcpSeed = (0x[0-9A-Fa-f]+);", open(SRC).read())
    return int(m.group(1), 16)


def test_reciprocal_seed_and_newton_steps():
    C = _seed_constant()
    bits = (np.uint32(127) << np.uint32(23)) | np.arange(1 << 23, dtype=np.uint32)
    d = bits.view(np.float32)
    r0 = (np.uint32(C) - bits).view(np.float32)
    err0 = np.abs(r0.astype(np.float64) * d.astype(np.float64) - 1.0)
    assert err0.max() < 0.0506
    # the three steps r <- r (2 - d r) as the kernel runs them: fp32 fused
    # multiply-adds e = fma(-d, r, 1), r = fma(r, e, r), each rounded once
    r = r0.astype(np.float64)
    d64 = d.astype(np.float64)
    for _ in range(3):
        e = (1.0 - d64 * r).astype(np.float32).astype(np.float64)
        r = (r + r * e).astype(np.float32).astype(np.float64)
    exact = 1.0 / d64
    ulp = np.spacing(exact.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(r - exact) / ulp) <= 2.0
