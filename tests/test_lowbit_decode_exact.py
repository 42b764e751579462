"""The fp16 arithmetic the low-bit GEMM decodes with is exact (no GPU).

The kernel turns a packed code u = q + 2^(b-1) and a group's E4M3 scale sigma
into the fp16 operand q * sigma / 16 with one fused multiply-add on fp16
values: t = 1024 + u (the code under the exponent of 1024), s = sigma / 16,
c = fp16(s * -(1024 + 2^(b-1))), result = fp16(t * s + c). It widens an
activation code x the same way: fp16(1024 + (x + 128)) - 1152. The GEMM is
only as exact as these steps, so every code and every finite non-negative
E4M3 scale is checked here with IEEE fp16 (NumPy), the fused step rounded
once from the exact float64 value.
"""

import numpy as np
import pytest

import oracle as O


def _f16(v):
    return np.asarray(v, dtype=np.float64).astype(np.float16).astype(np.float64)


@pytest.mark.parametrize("bits", [4, 6])
def test_weight_decode_is_exact_for_every_code_and_scale(bits):
    bias = 2 ** (bits - 1)
    sigma = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))   # 0 .. 448, every finite code
    u = np.arange(2 ** bits, dtype=np.float64)
    s = _f16(sigma / 16.0)
    assert np.array_equal(s, sigma / 16.0)                    # sigma / 16 is an fp16
    c = _f16(s * -(1024.0 + bias))
    assert np.array_equal(c, s * -(1024.0 + bias))            # the offset term is exact too
    t = _f16(1024.0 + u)
    got = _f16(t[None, :] * s[:, None] + c[:, None])          # one rounding: the fma
    want = (u[None, :] - bias) * sigma[:, None] / 16.0
    assert np.array_equal(got, want)


def test_activation_widening_is_exact():
    x = np.arange(-128, 128, dtype=np.float64)
    t = _f16(1024.0 + (x + 128.0))
    assert np.array_equal(_f16(t - 1152.0), x)
