"""Plain, slow, obviously-correct CPU definition of the W8A8 ConvRot MoE block.

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the bench's
CPU-baseline leg, never by the product path.

Sources (web pages, cited by title and section):

* "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder", section
  "Quantization": every routed-expert matrix is rotated with ConvRot, then
  quantised to symmetric INT8 with nearest rounding and one FP32 scale per
  output row; rotation groups are 256 for gate/up and 64 for down; inference
  runs W8A8 ConvRot linears with BF16 outputs.
* "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were made":
  int8 ConvRot is a block Hadamard rotation, one scale per row, and 8-bit
  activations.
* "MLX Nucleus-Image", opening paragraph: 64 routed experts per layer with
  expert-choice routing; table "Conversion notes": expert-choice means each
  expert picks its top-C tokens and the outputs are scattered back, and the
  MoE experts use silu(gate) * up with gate in the first half.

Readings of what the pages leave open (each is fixed here once):

* Hadamard: Sylvester construction in natural order, no sign flips,
  normalised by 1/sqrt(g); applied block-diagonally along K (contiguous
  groups of g) as an explicit fp64 matrix product. Only g in
  {1, 4, 16, 64, 256} (powers of four) are accepted, so 1/sqrt(g) is a power
  of two.
* Symmetric INT8 with nearest rounding of a rotated row v (fp64):
  a = max|v|, s = fp32(a / 127) (the fp64 quotient rounded once to fp32),
  q = clamp(rne(v / s), -127, 127) with the quotient taken in fp64 and ties
  to even. A row whose s is 0 (an all-zero row, or one too small for fp32)
  gets all-zero codes.
* Activations: per-token dynamic scales, the same rotation and quantiser as
  the weights; so is the SwiGLU output h before the down projection (g = 64,
  one scale per (expert, token) row).
* Router score: per-token softmax over the experts, evaluated in fp64 and
  rounded once to fp32. Top-C ties go to the lower token index; the selected
  indices are stored in ascending token order.
* Dequant: fp32(acc) * (s_w * s_x), the scale product first, IEEE fp32.
* SwiGLU: h = (g / (1 + e)) * u in fp32 with e = fp32(exp(-g)) (the
  exponential correctly rounded to fp32, computed here through fp64).
* Down projection output: z = bf16(fp32(acc) * (s_d * s_h)), since each
  expert linear is a W8A8 ConvRot linear with BF16 outputs (Nucleus-Image,
  "Quantization"). The gate/up output is not rounded: it feeds SwiGLU inside
  the same fused step, in fp32.
* Combine: out32[t] += fp32(w * z) in fp32 over experts in ascending order,
  one bf16 round-to-nearest-even at the end; tokens no expert picked give 0.

Numeric inputs are NumPy arrays. bf16 tensors are passed as float32 arrays
holding bf16-representable values (NumPy has no bf16 type).
"""

from __future__ import annotations

import numpy as np

ALLOWED_GROUPS = (1, 4, 16, 64, 256)
QMAX = 127


# ---------------------------------------------------------------- rotation --
def hadamard(g: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix H_g (int64), natural order.

    H_1 = [1]; H_2n = [[H_n, H_n], [H_n, -H_n]].
    """
    if g < 1 or (g & (g - 1)) != 0:
        raise ValueError(f"Hadamard order must be a power of two, got {g}")
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < g:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_matrix(g: int) -> np.ndarray:
    """R_g = H_g / sqrt(g) in fp64 (symmetric and orthogonal)."""
    if g not in ALLOWED_GROUPS:
        raise ValueError(f"group must be one of {ALLOWED_GROUPS}, got {g}")
    return hadamard(g).astype(np.float64) / np.sqrt(np.float64(g))


def block_rotate(v: np.ndarray, g: int) -> np.ndarray:
    """v' = v . blockdiag(R_g, ..., R_g) along the last axis (fp64).

    The last axis K is split into K/g contiguous groups; each group (a row
    vector) is multiplied on the right by R_g.
    """
    v = np.asarray(v, dtype=np.float64)
    k = v.shape[-1]
    if k % g != 0:
        raise ValueError(f"K={k} is not a multiple of the group size {g}")
    r = rotation_matrix(g)
    grouped = v.reshape(-1, g)  # every contiguous group of g as one row
    return (grouped @ r).reshape(v.shape)


# ------------------------------------------------------------ quantisation --
def quantize_rows(v: np.ndarray):
    """Symmetric per-row INT8 of a rotated matrix [rows, K] (see the header).

    Returns (q int8 [rows, K], s float32 [rows]).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.max(np.abs(v), axis=-1) if v.shape[-1] else np.zeros(v.shape[:-1])
    s = (a / np.float64(QMAX)).astype(np.float32)
    q = np.zeros(v.shape, dtype=np.int8)
    nz = s != 0
    if np.any(nz):
        quot = v[nz] / s[nz].astype(np.float64)[..., None]
        q[nz] = np.clip(np.rint(quot), -QMAX, QMAX).astype(np.int8)
    return q, s


def rotquant(x: np.ndarray, g: int):
    """Rotate each row by blockdiag(R_g) (fp64) and quantise it per row.

    Serves the weights (offline, per output row), the activations (per
    token) and the SwiGLU output h before the down projection (g = 64).
    """
    return quantize_rows(block_rotate(x, g))


# --------------------------------------------------------- integer GEMM -----
def int_gemm(a_q: np.ndarray, b_q: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k a_q[m, k] * b_q[n, k], exact, as int64.

    The products and every partial sum are integers of magnitude at most
    K * 127^2, far below 2^53, so the fp64 matrix product is exact whatever
    its summation order; it is used here only as a fast exact integer dot
    product. The result must also fit the int32 accumulator of the method.
    """
    a = np.asarray(a_q)
    b = np.asarray(b_q)
    k = a.shape[-1]
    if b.shape[-1] != k:
        raise ValueError("inner dimensions differ")
    if k * QMAX * QMAX >= 2**53:
        raise ValueError("K too large for an exact fp64 integer product")
    acc = a.astype(np.float64) @ b.astype(np.float64).T
    acc = acc.astype(np.int64)
    if acc.size and np.max(np.abs(acc)) >= 2**31:
        raise OverflowError("accumulator exceeds int32")
    return acc


def dequant(acc: np.ndarray, s_w: np.ndarray, s_x: np.ndarray) -> np.ndarray:
    """y[m, n] = fp32(acc[m, n]) * (s_w[n] * s_x[m]), IEEE fp32 operations."""
    acc32 = np.asarray(acc).astype(np.float32)
    scale = np.asarray(s_x, np.float32)[:, None] * np.asarray(s_w, np.float32)[None, :]
    return (acc32 * scale).astype(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returned as fp32.

    bf16 keeps the top 16 bits of the fp32 pattern: add half of the dropped
    range plus the tie-to-even bit, then truncate. NaN/Inf are not expected.
    """
    bits = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return rounded.view(np.float32)


def w8a8_linear_from_codes(x_q, s_x, w_q, s_w) -> np.ndarray:
    """The linear given quantised inputs: Y = bf16(fp32(acc) * (s_w * s_x))."""
    return bf16_round(dequant(int_gemm(x_q, w_q), s_w, s_x))


def w8a8_linear(x: np.ndarray, w_q: np.ndarray, s_w: np.ndarray, g: int) -> np.ndarray:
    """W8A8 ConvRot linear: Y = bf16(fp32(acc) * (s_w * s_x)).

    x: [M, K] bf16 values; w_q: [N, K] int8 rotated codes; s_w: [N] fp32.
    """
    x_q, s_x = rotquant(x, g)
    return w8a8_linear_from_codes(x_q, s_x, w_q, s_w)


# --------------------------------------------------------------- routing ----
def router_softmax(logits: np.ndarray) -> np.ndarray:
    """S[t, e] = softmax over experts of the token's logits, fp64 -> fp32."""
    l64 = np.asarray(logits, dtype=np.float64)
    m = np.max(l64, axis=-1, keepdims=True)
    e = np.exp(l64 - m)
    return (e / np.sum(e, axis=-1, keepdims=True)).astype(np.float32)


def expert_choice_topc(scores: np.ndarray, c: int):
    """Each expert picks the C tokens with the largest score.

    scores: [T, E] fp32. Ties go to the lower token index, i.e. the first C
    of a stable sort by (-score, t). Returns idx int32 [E, C] (ascending
    token order per expert) and w fp32 [E, C] = scores[idx[e, c], e].
    """
    s = np.asarray(scores, dtype=np.float32)
    t, n_exp = s.shape
    if not 0 <= c <= t:
        raise ValueError("capacity C must satisfy 0 <= C <= T")
    idx = np.zeros((n_exp, c), dtype=np.int32)
    w = np.zeros((n_exp, c), dtype=np.float32)
    for e in range(n_exp):
        order = np.argsort(-s[:, e], kind="stable")
        chosen = np.sort(order[:c])
        idx[e] = chosen
        w[e] = s[chosen, e]
    return idx, w


# ----------------------------------------------------------------- SwiGLU ---
def silu_f32(g: np.ndarray) -> np.ndarray:
    """silu(g) = g / (1 + exp(-g)) in fp32, exp correctly rounded to fp32."""
    g32 = np.asarray(g, dtype=np.float32)
    with np.errstate(over="ignore"):
        e = np.exp(-g32.astype(np.float64)).astype(np.float32)
    return (g32 / (np.float32(1) + e)).astype(np.float32)


def swiglu_from_codes(x_q, s_x, wgu_q, s_gu) -> np.ndarray:
    """One expert's gate/up linear given quantised inputs, then SwiGLU:
    y = fp32(acc) * (s_gu * s_x); h = silu(y[:, :f]) * y[:, f:] (fp32)."""
    y = dequant(int_gemm(x_q, wgu_q), s_gu, s_x)
    f = y.shape[1] // 2
    return (silu_f32(y[:, :f]) * y[:, f:]).astype(np.float32)


def down_from_codes(h_q, s_h, wd_q, s_d) -> np.ndarray:
    """One expert's down projection given quantised inputs: a W8A8 linear
    with BF16 output, z = bf16(fp32(acc) * (s_d * s_h))."""
    return w8a8_linear_from_codes(h_q, s_h, wd_q, s_d)


# --------------------------------------------------------------- combine ----
def combine_f32(t: int, idx: np.ndarray, w: np.ndarray, z: dict) -> np.ndarray:
    """Router-weighted sum before the final rounding: out32[idx[e, c]] +=
    fp32(w[e, c] * z[e][c]) in fp32, experts in ascending order.

    z maps expert e to its [C, d] bf16 outputs (as fp32); experts missing
    from z contribute nothing. Returns out32 [t, d] fp32.
    """
    d = next(iter(z.values())).shape[1] if z else 0
    out32 = np.zeros((t, d), dtype=np.float32)
    for e in sorted(z):
        rows = idx[e]
        # rows are distinct within an expert, so fancy-index += is exact;
        # the product w*z is rounded to fp32, then added in fp32
        out32[rows] = out32[rows] + (w[e][:, None] * z[e]).astype(np.float32)
    return out32


def combine(t: int, idx: np.ndarray, w: np.ndarray, z: dict) -> np.ndarray:
    """The router-weighted combine with its one bf16 rounding: Y [t, d] as
    fp32 holding bf16 values (see combine_f32)."""
    return bf16_round(combine_f32(t, idx, w, z))


# -------------------------------------------------------------- MoE block ---
def moe_block(x, logits, wgu_q, s_gu, wd_q, s_d, c, g_gu=256, g_d=64,
              experts=None, keep=False, out_tokens=None):
    """Expert-choice W8A8 ConvRot MoE block.

    x: [T, d] bf16 values; logits: [T, E] bf16 values;
    wgu_q: [E, 2f, d] int8 (rows 0..f-1 gate, f..2f-1 up), s_gu: [E, 2f];
    wd_q: [E, d, f] int8, s_d: [E, d]; c: tokens per expert.
    ``experts`` restricts the combine to a subset of experts (used to time a
    bounded sample); ``out_tokens`` evaluates only the output rows of those
    tokens (each row depends only on its own token, so the expert rows of
    other tokens are left 0 and so are their outputs); ``keep`` returns the
    intermediates as a dict.

    Returns Y as fp32 holding bf16 values [T, d] (and the dict if keep).
    """
    x = np.asarray(x, dtype=np.float32)
    t, d = x.shape
    n_exp = wgu_q.shape[0]
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
        h = swiglu_from_codes(x_q[rows], s_x[rows], wgu_q[e], s_gu[e])
        h_q, s_h = rotquant(h, g_d)
        z = np.zeros((c, d), dtype=np.float32)
        z[sel] = down_from_codes(h_q, s_h, wd_q[e], s_d[e])
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
