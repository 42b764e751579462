"""Checks of run-time INT8 codes against the oracle's definition.

The activation codes (and the codes of h before the down projection) come
from an fp32 rotation on the GPU, while the oracle's definition rotates with
an explicit fp64 Hadamard matrix and divides in fp64 ("Nucleus-Image INT8
Convrot Experts + FP8 Text Encoder", section "Quantization": symmetric INT8
with nearest rounding, one FP32 scale per row). A GPU code may therefore
differ from the definition's by one, and only where the exact quotient v'/s
lies within the fp32 error of a half-integer. The budget: at most 1e-4 of the
codes off by one (at least 8 allowed in small cases), none off by more.

The error bound per row: the fp32 butterflies of a group add at most
log2(g) roundings of 2^-24 times the group's |.|-sum / sqrt(g) to each
rotated value (``input_err`` adds what the input itself may differ by, e.g.
CUDA expf in h); the scale and the reciprocal add a few roundings of 2^-24.
"""

from __future__ import annotations

import numpy as np

import oracle as O

BUDGET = 1e-4


def rotation_error_bound(x64: np.ndarray, g: int, input_err: float = 0.0) -> np.ndarray:
    """Per row: a bound on |fp32 rotation - exact rotation| of any element."""
    rows, k = x64.shape
    stages = max(int(np.log2(g)), 0)
    grp = np.abs(x64).reshape(rows, k // g, g).sum(-1)  # [rows, groups]
    return ((stages + input_err) * 2.0 ** -24 * grp.max(-1) / np.sqrt(g)
            + 2.0 ** -149)


def check_codes(q_gpu: np.ndarray, s_gpu: np.ndarray, x: np.ndarray, g: int,
                input_err: float = 0.0, budget: float = BUDGET):
    """q_gpu [rows, K] int8, s_gpu [rows] fp32 from the GPU's fp32 path for
    input rows x (fp32/bf16 values) rotated in groups of g. Returns
    (flips, codes, q_ref, s_ref)."""
    x64 = np.asarray(x, dtype=np.float64)
    v = O.block_rotate(x64, g)
    q_ref, s_ref = O.quantize_rows(v)
    eps = rotation_error_bound(x64, g, input_err)  # [rows]
    a = np.abs(v).max(-1)
    # scales: s_gpu = fp32(a32 / 127) with |a32 - a| <= eps
    tol_s = eps / 127.0 + np.spacing(np.maximum(s_ref, np.float32(2.0 ** -126))).astype(np.float64)
    ds = np.abs(s_gpu.astype(np.float64) - s_ref.astype(np.float64))
    bad_s = np.nonzero(ds > 2 * tol_s)[0]
    assert bad_s.size == 0, f"scale outside its bound in rows {bad_s[:8]}"
    dq = q_gpu.astype(np.int32) - q_ref.astype(np.int32)
    assert np.abs(dq).max(initial=0) <= 1, "a code is off by more than one"
    r, c = np.nonzero(dq)
    if r.size:
        s64 = s_ref.astype(np.float64)[r]
        z = v[r, c] / s64
        dist = np.abs(np.abs(z - np.floor(z)) - 0.5)
        # deviation of the GPU's pre-rounding value from v'/s: the rotation
        # error of v' and of the absmax, and ~3 fp32 roundings of |v'/s|
        delta = 127.0 * (2 * eps[r] / np.maximum(a[r], 1e-300)) + np.abs(z) * 4 * 2.0 ** -24
        far = dist > 2 * delta
        assert not far.any(), (f"{int(far.sum())} codes differ from the definition away from a "
                               f"half-integer (first at row {r[far][0]}, col {c[far][0]})")
    flips = int(r.size)
    # the budget is a rate; small cases get a floor of 8 (one row whose absmax
    # makes many quotients exact half-integers can flip several codes, each of
    # them checked above to sit at a half-integer)
    assert flips <= max(8, budget * q_gpu.size), f"{flips} flips in {q_gpu.size} codes"
    return flips, q_gpu.size, q_ref, s_ref
