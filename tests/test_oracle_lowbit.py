"""Pins for the oracle's W4A8 / W6A8 formats (no GPU).

Definition: "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they
were made" (6-bit / 4-bit weights in the rotated basis, an FP8 scale per group
of 16, 8-bit activations); the readings are in oracle/lowbit_oracle.py.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from tests.golden import read_fixture


# ------------------------------------------------------------------ E4M3 ----
def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256)
    ours = O.e4m3_decode(codes)
    lib = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(lib)
    assert np.array_equal(ours[fin], lib[fin])
    assert np.isnan(ours).sum() == 2  # 0x7F and 0xFF


def test_e4m3_by_hand():
    assert O.e4m3_decode(0x7E) == 448.0
    assert O.e4m3_decode(0x01) == 2.0 ** -9
    assert O.e4m3_decode(0x08) == 2.0 ** -6  # smallest normal
    assert O.e4m3_decode(0x38) == 1.0
    assert O.e4m3_decode(0xB8) == -1.0
    enc = lambda v: int(O.e4m3_encode(np.float64(v)))
    assert enc(448) == 0x7E and enc(460) == 0x7E and enc(1e9) == 0x7E  # saturates
    assert enc(2.0 ** -10) == 0x00          # halfway 0 / 2^-9: the even code
    assert enc(3 * 2.0 ** -10) == 0x02      # halfway 2^-9 / 2^-8: the even code
    assert enc(17) == 0x58                  # halfway 16 / 18: 16 (mantissa 0)
    assert enc(19) == 0x5A                  # halfway 18 / 20: 20 (mantissa 2)
    assert enc(6.857142857142857) == 0x4E   # nearer 7.0 than 6.5


def test_e4m3_encode_matches_torch_rounding(rng):
    v = np.concatenate([np.abs(rng.standard_normal(20000)) * 60,
                        rng.random(5000) * 2.0 ** -6,
                        rng.random(5000) * 448]).astype(np.float32)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v.astype(np.float64)), lib)


def test_e4m3_encode_brute_force(rng):
    table = [(c, Fraction(float(O.e4m3_decode(c)))) for c in range(0x7F)]
    for v in list(rng.random(300) * 500) + [2.0 ** -12, 0.0, 447.9, 432.0, 416.0]:
        fv = Fraction(float(v))
        best = min(table, key=lambda cv: (abs(cv[1] - fv), cv[0] % 2))
        if fv > 448:
            best = (0x7E, None)
        assert int(O.e4m3_encode(np.float64(v))) == best[0], v


# ------------------------------------------------------------ quantiser -----
@pytest.mark.parametrize("bits", [4, 6])
def test_worked_rows(bits):
    fx = read_fixture("lowbit_worked.txt")
    v = np.array(fx[f"w{bits}_input"][0])
    q, sig, s_r = O.quantize_rows_lowbit(v[None], bits)
    assert s_r[0] == np.float32(fx[f"w{bits}_s_r"][0][0])
    assert sig[0].tolist() == [int(c) for c in fx[f"w{bits}_sigma"][0]]
    assert q[0].tolist() == [int(c) for c in fx[f"w{bits}_codes"][0]]


def _nearest_f32(fr):
    """The fp32 value nearest to the rational fr >= 0 (ties to even)."""
    lo = np.float32(float(fr))
    cands = {lo, np.nextafter(lo, np.float32(0)), np.nextafter(lo, np.float32(np.inf))}
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - fr),
                                     int(np.array(c).view(np.uint32)) & 1))


@pytest.mark.parametrize("bits", [4, 6])
def test_quantiser_brute_force(bits, rng):
    qmax = 2 ** (bits - 1) - 1
    v = rng.standard_normal((3, 48)) * np.array([[0.02], [1.0], [3e-5]])
    v[0, 16:32] *= 1e-3                       # a group far below the row maximum
    v[2, 32:] = 0.0                           # an all-zero group
    v = v.astype(np.float32).astype(np.float64)
    q, sig, s_r = O.quantize_rows_lowbit(v, bits)
    table = [(c, Fraction(float(O.e4m3_decode(c)))) for c in range(0x7F)]
    for r in range(v.shape[0]):
        a = max(Fraction(abs(float(x))) for x in v[r])
        assert s_r[r] == _nearest_f32(a / (qmax * 448))
        sr = Fraction(float(s_r[r]))
        for j in range(3):
            grp = v[r, 16 * j:16 * j + 16]
            aj = max(Fraction(abs(float(x))) for x in grp)
            ratio = aj / (qmax * sr)
            want = 0x7E if ratio > 448 else min(
                table, key=lambda cv: (abs(cv[1] - ratio), cv[0] % 2))[0]
            assert int(sig[r, j]) == want
            step = sr * Fraction(float(O.e4m3_decode(want)))
            for i, x in enumerate(grp):
                if step == 0:
                    assert q[r, 16 * j + i] == 0
                    continue
                z = Fraction(float(x)) / step
                best = min(range(-qmax, qmax + 1), key=lambda c: (abs(z - c), c % 2))
                assert q[r, 16 * j + i] == best


@pytest.mark.parametrize("bits", [4, 6])
def test_quantiser_properties(bits, rng):
    qmax = 2 ** (bits - 1) - 1
    v = O.block_rotate(rng.standard_normal((64, 512)) * 0.02, 256)
    q, sig, s_r = O.quantize_rows_lowbit(v, bits)
    assert np.abs(q).max() <= qmax
    assert np.all((sig == 0x7E).any(axis=1))   # the row maximum's group takes 448
    w = O.dequant_weights_lowbit(q, sig, s_r)
    step = np.repeat(s_r.astype(np.float64)[:, None] * O.e4m3_decode(sig), 16, axis=1)
    a_g = np.repeat(np.abs(v).reshape(64, -1, 16).max(-1), 16, axis=1)
    inside = np.abs(v) <= (qmax + 0.5) * step
    err = np.abs(v - w)
    assert np.all(err[inside] <= step[inside] / 2 * (1 + 1e-12))
    # clamped elements lose at most what the group maximum exceeds the grid
    assert np.all(err[~inside] <= (a_g - qmax * step)[~inside] * (1 + 1e-12))
    if bits == 4:
        assert inside.all()  # a 4-bit group's maximum never passes 7.5 steps


def test_zero_rows_and_tiny_rows():
    v = np.zeros((2, 32))
    v[1, 3] = 2.0 ** -160  # s_r rounds to 0 in fp32
    q, sig, s_r = O.quantize_rows_lowbit(v, 4)
    assert np.all(q == 0) and np.all(sig == 0) and np.all(s_r == 0)


# -------------------------------------------------------------- linears -----
def test_acc_is_exact(rng):
    x_q = rng.integers(-127, 128, size=(3, 32)).astype(np.int8)
    q = rng.integers(-31, 32, size=(4, 32)).astype(np.int8)
    sig = rng.integers(0, 0x7F, size=(4, 2)).astype(np.uint8)
    acc = O.lowbit_acc(x_q, q, sig)
    for m in range(3):
        for n in range(4):
            want = sum(Fraction(int(x_q[m, k])) * int(q[n, k])
                       * Fraction(float(O.e4m3_decode(sig[n, k // 16]))) for k in range(32))
            assert Fraction(float(acc[m, n])) == want


def test_unit_group_scales_reduce_to_integer_gemm(rng):
    """sigma = 1.0 everywhere: the low-bit linear is the int8 linear of the
    same codes and row scales (a case the int8 oracle already pins)."""
    x_q = rng.integers(-127, 128, size=(5, 64)).astype(np.int8)
    s_x = (rng.random(5) * 0.1).astype(np.float32)
    q = rng.integers(-7, 8, size=(6, 64)).astype(np.int8)
    s_r = (rng.random(6) * 0.01).astype(np.float32)
    sig = np.full((6, 4), 0x38, dtype=np.uint8)
    assert np.array_equal(O.lowbit_linear_from_codes(x_q, s_x, q, sig, s_r),
                          O.w8a8_linear_from_codes(x_q, s_x, q, s_r))


@pytest.mark.parametrize("bits,tol", [(4, 0.13), (6, 0.04)])
def test_linear_close_to_unquantised(bits, tol, rng):
    x = rng.standard_normal((32, 512)).astype(np.float32)
    x[:, 7] *= 20
    w = (rng.standard_normal((48, 512)) * 0.02).astype(np.float32)
    q, sig, s_r = O.rotquant_lowbit(w, 256, bits)
    y = O.lowbit_linear(x, q, sig, s_r, 256)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < tol
    # the int8 format of the same weights is closer, the 6-bit closer than the 4-bit
    q8, s8 = O.rotquant(w, 256)
    y8 = O.w8a8_linear(x, q8, s8, 256)
    assert np.linalg.norm(y8 - ref) < np.linalg.norm(y - ref)


def test_weights_decode_to_the_rotated_weights(rng):
    w = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    v = O.block_rotate(w, 64)
    for bits in (4, 6):
        q, sig, s_r = O.rotquant_lowbit(w, 64, bits)
        wd = O.dequant_weights_lowbit(q, sig, s_r)
        # rotating back (R is symmetric and orthogonal) recovers w within the steps
        back = O.block_rotate(wd, 64)
        assert np.abs(back - w).max() < np.abs(v).max() / (2 ** (bits - 1) - 1)


# ------------------------------------------------------------- MoE block ----
def test_moe_lowbit_matches_int8_block_when_formats_coincide(rng):
    """With sigma = 1.0 and codes within +-7 the two formats decode to the same
    weights, and the low-bit block must reproduce the pinned int8 block."""
    t, d, f, e, c = 48, 64, 32, 3, 16
    x = torch.from_numpy(rng.standard_normal((t, d)).astype(np.float32)).bfloat16().float().numpy()
    logits = torch.from_numpy(rng.standard_normal((t, e)).astype(np.float32)).bfloat16().float().numpy()
    gu_q = rng.integers(-7, 8, size=(e, 2 * f, d)).astype(np.int8)
    gu_s = (rng.random((e, 2 * f)) * 0.01).astype(np.float32)
    dn_q = rng.integers(-7, 8, size=(e, d, f)).astype(np.int8)
    dn_s = (rng.random((e, d)) * 0.01).astype(np.float32)
    ones_gu = np.full((e, 2 * f, d // 16), 0x38, np.uint8)
    ones_dn = np.full((e, d, f // 16), 0x38, np.uint8)
    y_low = O.moe_block_lowbit(x, logits, (gu_q, ones_gu, gu_s), (dn_q, ones_dn, dn_s), c,
                               g_gu=16, g_d=16)
    y_int = O.moe_block(x, logits, gu_q, gu_s, dn_q, dn_s, c, g_gu=16, g_d=16)
    assert np.array_equal(y_low, y_int)


@pytest.mark.parametrize("bits,tol", [(4, 0.3), (6, 0.1)])
def test_moe_lowbit_single_expert_is_dense_mlp(bits, tol, rng):
    t, d, f = 32, 256, 128
    x = torch.from_numpy(rng.standard_normal((t, d)).astype(np.float32)).bfloat16().float().numpy()
    logits = np.zeros((t, 1), np.float32)   # one expert: every router weight is 1
    wg = (rng.standard_normal((2 * f, d)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((d, f)) * 0.05).astype(np.float32)
    gu = tuple(a[None] for a in O.rotquant_lowbit(wg, 256, bits))
    dn = tuple(a[None] for a in O.rotquant_lowbit(wd, 64, bits))
    y = O.moe_block_lowbit(x, logits, gu, dn, t)
    y64 = x.astype(np.float64) @ wg.T.astype(np.float64)
    h = y64[:, :f] / (1 + np.exp(-y64[:, :f])) * y64[:, f:]
    ref = h @ wd.T.astype(np.float64)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < tol
