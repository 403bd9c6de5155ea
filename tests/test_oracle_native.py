"""The oracle's C row quantizers (oracle/quant_rows.c) give the same values as
its numpy quantizers, bit for bit, on every kind of block: ordinary values at
several magnitudes, all-zero blocks, blocks far below the tensor's amax (NVFP4
zero block scales), saturating blocks and exact rounding ties."""

import numpy as np
import pytest

from oracle import moe_oracle as O
from oracle import native


def _cases(K):
    rng = np.random.default_rng(11)
    out = []
    for scale in (1e-3, 0.05, 1.0, 37.0, 3e4):
        out.append(O.round_bf16(rng.normal(size=(67, K)) * scale))
    v = O.round_bf16(rng.normal(size=(40, K)))
    v[0] = 0.0
    v[1, :16] = 0.0
    v[2] *= 1e-7                      # far below the amax of the tensor
    v[3, :32] = [6.0, 2.5, -0.75, 1.25] * 8   # ties at the e2m1 midpoints
    v[4, :32] = [448.0, 272.0 / 512, 1.9921875, -510 / 256] * 8
    out.append(v)
    return out


@pytest.mark.skipif(native.load() is None, reason="no C compiler for the oracle helper")
@pytest.mark.parametrize("dtype", ["mxfp8", "nvfp4"])
def test_native_matches_numpy(dtype):
    for v in _cases(512):
        gs = [None]
        if dtype == "nvfp4":
            gs = [None, O.nvfp4_global_scale(1.0), O.nvfp4_global_scale(np.abs(v).max() * 3)]
        for g in gs:
            a = O.quantize_dequantize(v, dtype, g)
            b = O.quantize_dequantize(v, dtype, g, native=False)
            assert np.array_equal(a, b)
            assert np.array_equal(np.signbit(a), np.signbit(b))
