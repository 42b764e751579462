"""Pins for the oracle's quantiser, integer GEMM, dequant and W8A8 linear (no GPU).

Definitions: "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder",
section "Quantization" (symmetric INT8, nearest rounding, one FP32 scale per
output row, W8A8 linears with BF16 outputs); "NitroFusion2 for ComfyUI:
int8, W6A8, W4A8", section "How they were made" (one scale per row, 8-bit
activations).
"""

import numpy as np
import pytest
import torch

from oracle import (bf16_round, block_rotate, dequant, fwht_f32, int_gemm, quantize_rows,
                    rotquant, w8a8_linear)
from tests.golden import read_fixture


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def test_worked_ties_to_even():
    fx = read_fixture("quant_ties.txt")
    q, s = quantize_rows(np.array(fx["input"]))
    assert s.tolist() == fx["scale"][0]
    assert q[0].tolist() == fx["codes"][0]


def test_worked_rotated_codes_g4():
    fx = read_fixture("rotation_g4.txt")
    q, s = rotquant(np.array(fx["input"]), 4)
    assert q[0].tolist() == fx["codes"][0]
    assert s[0] == np.float32(13) / np.float32(127)


def test_quantiser_bounds(rng):
    v = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 50, size=(64, 1))).astype(np.float32)
    q, s = quantize_rows(v)
    s64 = s.astype(np.float64)[:, None]
    assert np.all(np.abs(q.astype(np.int64)) <= 127)
    # nearest code up to the fp32 reciprocal: |v - s q| <= s (1/2 + 1e-4)
    assert np.all(np.abs(v - s64 * q) <= s64 * (0.5 + 1e-4))
    # the absmax element of every row gets a full-scale code
    j = np.argmax(np.abs(v), axis=1)
    assert np.all(np.abs(q[np.arange(64), j]) == 127)
    # the scale is absmax/127 as one fp32 division
    assert np.array_equal(s, np.max(np.abs(v), axis=1) / np.float32(127))


def test_quantiser_nearest_code_property(rng):
    """Every code is the nearest integer to the exact v / s, ties to even,
    except where v / s lies within 1e-4 of a half-integer (the fp32
    reciprocal may tip it); there it is one of the two neighbours."""
    v = rng.standard_normal((16, 64)).astype(np.float32)
    v[1, 3] = 0.0
    v[2, :8] = np.float32(127) * np.array([1, 0.5, 2.5, -2.5, 3.5, 1.5, -0.5, 126.5], np.float32) / 127
    q, s = quantize_rows(v)
    codes = np.arange(-127, 128)
    for i in range(v.shape[0]):
        for j in range(v.shape[1]):
            x = float(v[i, j]) / float(s[i])
            dist = np.abs(x - codes)
            best = codes[dist == dist.min()]
            frac = abs(abs(x - np.floor(x)) - 0.5)
            if frac > 1e-4:
                assert q[i, j] == (best[0] if len(best) == 1 else best[best % 2 == 0][0])
            else:
                assert q[i, j] in (np.floor(x), np.ceil(x))


def test_zero_and_tiny_rows():
    v = np.zeros((3, 8), np.float32)
    v[1, 2] = np.float32(2.0 ** -121)   # below the 2^-120 floor: treated as zero
    v[2, 2] = np.float32(2.0 ** -119)
    q, s = quantize_rows(v)
    assert np.all(q[:2] == 0) and np.all(s[:2] == 0)
    assert q[2, 2] == 127 and s[2] == np.float32(2.0 ** -119) / np.float32(127)


def test_int_gemm_triple_loop(rng):
    a = rng.integers(-127, 128, size=(5, 7)).astype(np.int8)
    b = rng.integers(-127, 128, size=(3, 7)).astype(np.int8)
    got = int_gemm(a, b)
    for m in range(5):
        for n in range(3):
            assert got[m, n] == sum(int(a[m, k]) * int(b[n, k]) for k in range(7))


def test_int_gemm_extremes_and_overflow():
    k = 2048
    a = np.full((2, k), 127, np.int8)
    b = np.full((2, k), -127, np.int8)
    assert int_gemm(a, b)[0, 0] == -k * 127 * 127  # 33,032,192 fits int32
    k_big = 2**31 // (127 * 127) + 1
    with pytest.raises(OverflowError):
        int_gemm(np.full((1, k_big), 127, np.int8), np.full((1, k_big), 127, np.int8))


def test_dequant_indexing_brute_force(rng):
    acc = rng.integers(-2**24, 2**24, size=(3, 5))
    s_w = rng.uniform(1e-4, 1e-2, size=5).astype(np.float32)
    s_x = rng.uniform(1e-2, 1.0, size=3).astype(np.float32)
    y = dequant(acc, s_w, s_x)
    for m in range(3):
        for n in range(5):
            assert y[m, n] == np.float32(acc[m, n]) * (s_w[n] * s_x[m])


def test_bf16_round_matches_library(rng):
    x = (rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000)).astype(np.float32)
    bits = x.view(np.uint32)
    ties = ((bits & 0xFFFF0000) | 0x8000).view(np.float32)  # exact half-way cases
    for arr in (x, ties):
        ref = torch.from_numpy(arr).to(torch.bfloat16).float().numpy()
        assert np.array_equal(bf16_round(arr), ref)


def _linear_error_bound(x, w, g, y):
    """Rigorous bound on |Y - X W^T| for the W8A8 ConvRot linear."""
    xr, wr = fwht_f32(x, g).astype(np.float64), fwht_f32(w, g).astype(np.float64)
    xq, sx = quantize_rows(xr)
    wq, sw = quantize_rows(wr)
    w_hat = wq * sw.astype(np.float64)[:, None]
    half = 0.5 + 1e-4
    # quantisation: |x'.w' - x_hat.w_hat| <= sum|x'| |w' - w_hat| + sum |w_hat| |x' - x_hat|
    bound = (np.abs(xr).sum(1)[:, None] * (sw.astype(np.float64)[None, :] * half)
             + (sx.astype(np.float64)[:, None] * half) * np.abs(w_hat).sum(1)[None, :])
    # fp32 rotation of x and w: log2(g) roundings of at most the group's |.|-sum
    st = max(int(np.log2(g)), 0) * 2.0 ** -24 / np.sqrt(g)
    ex = st * np.abs(x.astype(np.float64)).reshape(x.shape[0], -1, g).sum(-1).max(-1)
    ew = st * np.abs(w.astype(np.float64)).reshape(w.shape[0], -1, g).sum(-1).max(-1)
    bound += (ex[:, None] * np.abs(wr).sum(1)[None, :] + np.abs(xr).sum(1)[:, None] * ew[None, :])
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    # fp32 dequant (3 roundings) and the final bf16 rounding
    slack = np.abs(ref + bound) * (2.0 ** -8 + 4 * 2.0 ** -24) + 1e-30
    return np.abs(y - ref), bound + slack


@pytest.mark.parametrize("g", [1, 4, 16, 64, 256])
def test_linear_within_quantisation_bound(g, rng):
    m, n, k = 32, 24, 512
    x = rng.standard_normal((m, k)).astype(np.float32)
    x[:, rng.choice(k, 5, replace=False)] *= 20.0
    x = _bf16(x)
    w = _bf16(rng.standard_normal((n, k)) * 0.02)
    wq, sw = rotquant(w, g)
    y = w8a8_linear(x, wq, sw, g)
    err, bound = _linear_error_bound(x, w, g, y)
    assert np.all(err <= bound)


def test_rotation_reduces_outlier_error(rng):
    """Spreading outlier channels over a group lowers the W8A8 error."""
    m, n, k = 64, 64, 1024
    x = rng.standard_normal((m, k)).astype(np.float32)
    x[:, rng.choice(k, 10, replace=False)] *= 20.0
    x = _bf16(x)
    w = _bf16(rng.standard_normal((n, k)) * 0.02)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    errs = {}
    for g in (1, 256):
        wq, sw = rotquant(w, g)
        errs[g] = np.linalg.norm(w8a8_linear(x, wq, sw, g) - ref)
    assert errs[256] < 0.5 * errs[1]
