"""CPU definition of the W4A8 / W6A8 formats in the rotated basis.

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the bench's
CPU-baseline leg, never by the product path.

Source: "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were
made": besides int8 ConvRot, the linears come as 6-bit or 4-bit weights in
the rotated basis with an FP8 scale for every group of 16 weights, and 8-bit
activations.

Readings of what the page leaves open (each is fixed here once):

* Rotated basis: the int8 format's block Hadamard rotation (see
  convrot_oracle), with the same groups (256 for dense linears and the
  experts' gate/up, 64 for the down projection).
* Codes: symmetric, q in [-qmax, qmax] with qmax = 2^(b-1) - 1 (7 for 4-bit,
  31 for 6-bit), nearest rounding with ties to even, like the int8 codes;
  -2^(b-1) is never produced.
* FP8: E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
  subnormals, largest finite value 448, no infinities).
* Two scale levels: an FP8 number alone cannot cover a row's range (weights
  of typical size would fall into E4M3's subnormals), so each row keeps the
  int8 format's FP32 scale and the FP8 scale of a group is relative to it.
  For a rotated row v (fp64) with group maxima a_j = max |v| over group j
  (16 consecutive elements along K) and a = max_j a_j:
    s_r   = fp32(a / (qmax * 448))          (fp64 quotient rounded once)
    sigma = e4m3(a_j / (qmax * s_r))        (nearest, ties to the even
                                             code, at most 448)
    q     = clamp(rne(v / (s_r * sigma)), -qmax, qmax)   (fp64 quotient)
  A row with s_r = 0 and a group with sigma = 0 get zero codes. The weight
  the kernel decodes is s_r * sigma * q.
* Activations: per-token INT8 exactly as in the int8 format.
* Linear: y[m, n] = fp32(acc) * (s_r[n] * s_x[m]) with
  acc = sum_k x_q[m, k] * sigma[n, k / 16] * q[n, k] taken exactly; BF16
  output.

Exactness of acc in fp64: every term is a multiple of 2^-9 (the smallest
E4M3 step) of magnitude below 127 * 448 * 31 < 2^21, so for K < 2^23 every
partial sum is a multiple of 2^-9 below 2^44 and the fp64 matrix product is
exact in any summation order.
"""

from __future__ import annotations

import numpy as np

from .convrot_oracle import (
    bf16_round,
    block_rotate,
    combine_f32,
    expert_choice_topc,
    rotquant,
    router_softmax,
    silu_f32,
)

GROUP = 16          # weights per FP8 scale
E4M3_MAX = 448.0
LOWBIT_BITS = (4, 6)


def qmax_of(bits: int) -> int:
    if bits not in LOWBIT_BITS:
        raise ValueError(f"bits must be one of {LOWBIT_BITS}, got {bits}")
    return 2 ** (bits - 1) - 1


# -------------------------------------------------------------- E4M3 --------
def e4m3_decode(code) -> np.ndarray:
    """Value of E4M3 byte(s) as fp64: sign, exponent e (bias 7), mantissa m:
    e = 0 gives m * 2^-9 (subnormal), else (1 + m/8) * 2^(e - 7);
    e = 15 with m = 7 is NaN."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_POS_CODES = np.arange(0x7F, dtype=np.int64)      # 0x00 .. 0x7E: every finite value >= 0
_POS_VALUES = e4m3_decode(_POS_CODES)             # increasing


def e4m3_encode(v) -> np.ndarray:
    """Nearest finite non-negative E4M3 code to each v >= 0 (fp64), ties to
    the even code, v above 448 saturating to 448. Returns uint8."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("e4m3_encode takes non-negative numbers")
    hi = np.clip(np.searchsorted(_POS_VALUES, v, side="left"), 0, len(_POS_VALUES) - 1)
    lo = np.clip(hi - 1, 0, None)
    d_lo = np.abs(v - _POS_VALUES[lo])
    d_hi = np.abs(_POS_VALUES[hi] - v)
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    pick = np.where(tie, np.where(_POS_CODES[lo] % 2 == 0, lo, hi), pick)
    return _POS_CODES[pick].astype(np.uint8)


# --------------------------------------------------------- quantisation -----
def quantize_rows_lowbit(v: np.ndarray, bits: int):
    """Two-level low-bit quantisation of rotated rows v [rows, K] (fp64).

    Returns (q int8 [rows, K], sigma uint8 E4M3 codes [rows, K/16],
    s_r float32 [rows]); see the header for the definition.
    """
    qmax = qmax_of(bits)
    v = np.asarray(v, dtype=np.float64)
    rows, k = v.shape
    if k % GROUP:
        raise ValueError(f"K={k} is not a multiple of {GROUP}")
    a_g = np.abs(v).reshape(rows, k // GROUP, GROUP).max(-1) if k else np.zeros((rows, 0))
    a = a_g.max(-1) if k else np.zeros(rows)
    s_r = (a / np.float64(qmax * E4M3_MAX)).astype(np.float32)
    s64 = s_r.astype(np.float64)
    sigma = np.zeros((rows, k // GROUP), dtype=np.uint8)
    nz = s_r != 0
    if np.any(nz):
        sigma[nz] = e4m3_encode(a_g[nz] / (qmax * s64[nz])[:, None])
    step = s64[:, None] * e4m3_decode(sigma)       # exact: 24-bit times 4-bit significands
    q = np.zeros((rows, k), dtype=np.int8)
    step_k = np.repeat(step, GROUP, axis=1)
    live = step_k != 0
    q[live] = np.clip(np.rint(v[live] / step_k[live]), -qmax, qmax).astype(np.int8)
    return q, sigma, s_r


def rotquant_lowbit(w: np.ndarray, g: int, bits: int):
    """Rotate weight rows by blockdiag(R_g) (fp64) and quantise them to the
    b-bit two-level format."""
    return quantize_rows_lowbit(block_rotate(w, g), bits)


def dequant_weights_lowbit(q, sigma, s_r) -> np.ndarray:
    """The weights the kernel decodes, s_r * sigma * q, exactly (fp64)."""
    q = np.asarray(q, dtype=np.float64)
    sig = np.repeat(e4m3_decode(sigma), GROUP, axis=-1)
    return np.asarray(s_r, np.float64)[..., None] * sig * q


def lowbit_acc(x_q, q, sigma) -> np.ndarray:
    """acc[m, n] = sum_k x_q[m, k] * sigma[n, k/16] * q[n, k], exact (fp64)."""
    x = np.asarray(x_q, dtype=np.float64)
    wq = np.asarray(q, dtype=np.float64) * np.repeat(e4m3_decode(sigma), GROUP, axis=-1)
    if x.shape[-1] != wq.shape[-1]:
        raise ValueError("inner dimensions differ")
    if x.shape[-1] >= 2 ** 23:
        raise ValueError("K too large for an exact fp64 product")
    return x @ wq.T


def lowbit_dequant(acc, s_r, s_x) -> np.ndarray:
    """y[m, n] = fp32(acc[m, n]) * (s_r[n] * s_x[m]), IEEE fp32 operations."""
    acc32 = np.asarray(acc).astype(np.float32)
    scale = np.asarray(s_x, np.float32)[:, None] * np.asarray(s_r, np.float32)[None, :]
    return (acc32 * scale).astype(np.float32)


def lowbit_linear_from_codes(x_q, s_x, q, sigma, s_r) -> np.ndarray:
    """The low-bit linear given quantised inputs, BF16 output."""
    return bf16_round(lowbit_dequant(lowbit_acc(x_q, q, sigma), s_r, s_x))


def lowbit_linear(x, q, sigma, s_r, g: int) -> np.ndarray:
    """WbA8 ConvRot linear: the activations rotated and quantised per token
    to INT8 (the int8 format's path), the weights in the b-bit format."""
    x_q, s_x = rotquant(x, g)
    return lowbit_linear_from_codes(x_q, s_x, q, sigma, s_r)


def lowbit_swiglu_from_codes(x_q, s_x, q, sigma, s_r) -> np.ndarray:
    """One expert's gate/up linear in the b-bit format, then SwiGLU:
    y = fp32(acc) * (s_r * s_x); h = silu(y[:, :f]) * y[:, f:] (fp32)."""
    y = lowbit_dequant(lowbit_acc(x_q, q, sigma), s_r, s_x)
    f = y.shape[1] // 2
    return (silu_f32(y[:, :f]) * y[:, f:]).astype(np.float32)


def moe_block_lowbit(x, logits, gu, dn, c, g_gu=256, g_d=64, experts=None,
                     keep=False, out_tokens=None):
    """The expert-choice MoE block with b-bit expert weights.

    gu = (q [E, 2f, d], sigma [E, 2f, d/16], s_r [E, 2f]) (gate rows first),
    dn = (q [E, d, f], sigma [E, d, f/16], s_r [E, d]). Routing, the
    activation and h quantisation and the combine are the int8 block's;
    only the expert linears read b-bit weights. ``experts``, ``out_tokens``
    and ``keep`` as in convrot_oracle.moe_block.
    """
    x = np.asarray(x, dtype=np.float32)
    t, d = x.shape
    n_exp = gu[0].shape[0]
    x_q, s_x = rotquant(x, g_gu)
    scores = router_softmax(logits)
    idx, w = expert_choice_topc(scores, c)
    inter = {"x_q": x_q, "s_x": s_x, "scores": scores, "idx": idx, "w": w,
             "h": {}, "h_q": {}, "s_h": {}, "z": {}}
    z_all = {}
    for e in (range(n_exp) if experts is None else experts):
        sel = np.arange(c)
        if out_tokens is not None:
            sel = np.nonzero(np.isin(idx[e], out_tokens))[0]
            if sel.size == 0:
                continue
        rows = idx[e][sel]
        h = lowbit_swiglu_from_codes(x_q[rows], s_x[rows], gu[0][e], gu[1][e], gu[2][e])
        h_q, s_h = rotquant(h, g_d)
        z = np.zeros((c, d), dtype=np.float32)
        z[sel] = lowbit_linear_from_codes(h_q, s_h, dn[0][e], dn[1][e], dn[2][e])
        z_all[e] = z
        if keep:
            inter["h"][e], inter["h_q"][e], inter["s_h"][e] = h, h_q, s_h
            inter["z"][e] = z
    out32 = combine_f32(t, idx, w, z_all) if z_all else np.zeros((t, d), np.float32)
    y_out = bf16_round(out32)
    if keep:
        inter["out32"] = out32
        return y_out, inter
    return y_out
