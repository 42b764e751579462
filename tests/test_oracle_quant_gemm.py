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

from fractions import Fraction

from oracle import (bf16_round, block_rotate, dequant, int_gemm, quantize_rows, rotquant,
                    w8a8_linear, w8a8_linear_from_codes)
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


def _nearest_f32(x: Fraction) -> np.float32:
    """The fp32 value nearest to the exact rational x (ties to even), found
    by comparing the neighbours of a candidate in exact arithmetic."""
    c = np.float32(float(x))
    best = None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - x)
        even = (int(np.float32(cand).view(np.uint32)) & 1) == 0
        if best is None or d < best[0] or (d == best[0] and even):
            best = (d, cand)
    return np.float32(best[1])


def test_quantiser_scale_is_fp32_of_absmax_over_127(rng):
    """s is the fp32 value nearest to the exact absmax / 127."""
    v = rng.standard_normal((40, 96)) * 10.0 ** rng.integers(-20, 20, (40, 1))
    _, s = quantize_rows(v)
    for i in range(v.shape[0]):
        a = max(Fraction(abs(float(x))) for x in v[i])
        assert s[i] == _nearest_f32(a / 127)


def test_quantiser_bounds(rng):
    v = rng.standard_normal((64, 256)) * rng.uniform(0.01, 50, size=(64, 1))
    q, s = quantize_rows(v)
    s64 = s.astype(np.float64)[:, None]
    assert np.all(np.abs(q.astype(np.int64)) <= 127)
    # nearest code of the fp64 quotient: |v - s q| <= s (1/2 + 127 * 2^-53)
    assert np.all(np.abs(v - s64 * q) <= s64 * (0.5 + 2.0 ** -46))
    # the absmax element of every row gets a full-scale code
    j = np.argmax(np.abs(v), axis=1)
    assert np.all(np.abs(q[np.arange(64), j]) == 127)


def test_quantiser_nearest_code_brute_force(rng):
    """Every code is the integer in [-127, 127] nearest to the exact v / s
    (ties to even), found by trying all 255 codes in exact arithmetic. The
    only allowed exception is a quotient within 127 * 2^-53 of a half-integer
    (the fp64 division may tip it); none occurs in these rows."""
    v = rng.standard_normal((12, 48))
    v[1, 3] = 0.0
    # exact half-integer quotients: the row's absmax is 127, so s = 1
    v[2, :9] = [127, 0.5, 2.5, -2.5, 3.5, 1.5, -0.5, 126.5, -126.5]
    # a row with absmax 1, so s = fp32(1/127) != 1/127: between
    # (k + 1/2) * s and (k + 1/2) / 127 the quotient by s and the quotient by
    # the unrounded absmax / 127 fall on different sides of k + 1/2
    v[3, :] = 0.0
    v[3, 0] = 1.0
    s_f32 = Fraction(float(np.float32(1.0 / 127.0)))
    for j, k in enumerate((100, 57, 3), start=1):
        lo, hi = sorted((Fraction(2 * k + 1, 2) * s_f32, Fraction(2 * k + 1, 2) / 127))
        v[3, j] = float((lo + hi) / 2)
        v[3, j + 3] = -float((lo + hi) / 2)
    q, s = quantize_rows(v)
    codes = range(-127, 128)
    for i in range(v.shape[0]):
        si = Fraction(float(s[i]))
        for j in range(v.shape[1]):
            x = Fraction(float(v[i, j])) / si
            dist = {c: abs(x - c) for c in codes}
            m = min(dist.values())
            best = [c for c in codes if dist[c] == m]
            want = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
            assert q[i, j] == want, (i, j, float(x))


def test_zero_and_tiny_rows():
    """s = fp32(a / 127) may be subnormal or 0 for a tiny row. Worked by hand:
    row 1: a = 2^-140, a / 127 = 2^-149 * 512/127 = 2^-149 * 4.03.. -> the
    subnormal s = 4 * 2^-149 = 2^-147; codes 2^-140 / s = 128 -> clamped to 127,
    2^-141 / s = 64, -2^-140 / s = -128 -> clamped to -127. Row 2: a = 2^-145, a / 127 = 2^-149 * 0.126 -> s = 0, codes 0."""
    v = np.zeros((3, 8))
    v[1, 2], v[1, 5], v[1, 6] = 2.0 ** -140, -(2.0 ** -141), -(2.0 ** -140)
    v[2, 0] = 2.0 ** -145
    q, s = quantize_rows(v)
    assert np.all(q[0] == 0) and s[0] == 0
    assert s[1] == np.float32(2.0 ** -147)
    assert q[1].tolist() == [0, 0, 127, 0, 0, -64, -127, 0]  # +-128 clamped to +-127
    assert np.all(q[2] == 0) and s[2] == 0


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
    xr, wr = block_rotate(x, g), block_rotate(w, g)
    xq, sx = quantize_rows(xr)
    wq, sw = quantize_rows(wr)
    w_hat = wq * sw.astype(np.float64)[:, None]
    half = 0.5 + 2.0 ** -46
    # quantisation: |x'.w' - x_hat.w_hat| <= sum|x'| |w' - w_hat| + sum |w_hat| |x' - x_hat|
    bound = (np.abs(xr).sum(1)[:, None] * (sw.astype(np.float64)[None, :] * half)
             + (sx.astype(np.float64)[:, None] * half) * np.abs(w_hat).sum(1)[None, :])
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    # fp64 rotation of bf16 data is exact up to fp64 rounding; fp32 dequant
    # (3 roundings) and the final bf16 rounding
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


def test_linear_from_codes_is_the_linear(rng):
    x = _bf16(rng.standard_normal((8, 256)))
    w = _bf16(rng.standard_normal((12, 256)) * 0.02)
    wq, sw = rotquant(w, 64)
    xq, sx = rotquant(x, 64)
    assert np.array_equal(w8a8_linear(x, wq, sw, 64), w8a8_linear_from_codes(xq, sx, wq, sw))
