"""Thin Python binding of libconvrot.so (the C ABI in include/convrot.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI. PyTorch is used for device memory (output and
workspace tensors) and for the current CUDA stream. There is no CPU or
PyTorch fallback: if the library is missing or the device is not an sm_100
part, the calls raise.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libconvrot.so")

CONVROT_OK = 0
CONVROT_ERR_INVALID_ARG = 1
CONVROT_ERR_UNSUPPORTED_DEVICE = 2
CONVROT_ERR_WORKSPACE_TOO_SMALL = 3
CONVROT_ERR_MISALIGNED = 4
CONVROT_ERR_CUDA = 5
CONVROT_ERR_TIMEOUT = 6
DTYPE_BF16 = 0
DTYPE_F32 = 1
LAYOUT_ROWS = 0
LAYOUT_TILES = 1


class ConvrotError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        extra = ""
        if status == CONVROT_ERR_CUDA:
            extra = f": {lib().convrot_last_cuda_error().decode()}"
        super().__init__(f"{where}: {status_string(status)}{extra} (status {status})")


class MoeLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("x_q", "s_x", "s_t", "idx", "w", "x_g", "s_g", "h", "h_q", "s_h", "hsync", "slot",
                 "z", "total")]


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "convrot_abi_version": (_I, []),
    "convrot_status_string": (ctypes.c_char_p, [_I]),
    "convrot_last_cuda_error": (ctypes.c_char_p, []),
    "convrot_device_check": (_I, []),
    "convrot_check_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "convrot_wait_selftest": (_I, [ctypes.c_ulonglong, _P, _P]),
    "convrot_count_wait_selftest": (_I, [ctypes.c_ulonglong, _P, _P, _P]),
    "convrot_swiglu_rq_units": (_I64, [_I64, _I64, _I64]),
    "convrot_rotquant": (_I, [_P, _I, _I64, _I64, _I, _P, _P, _P]),
    "convrot_quantize_weights": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "convrot_tiled_weight_bytes": (_I64, [_I64, _I64, _I64]),
    "convrot_quantize_weights_tiled": (_I, [_P, _I64, _I64, _I64, _I, _P, _P, _P]),
    "convrot_router_softmax": (_I, [_P, _I64, _I, _P, _P]),
    "convrot_topc": (_I, [_P, _I64, _I, _I64, _P, _P, _P, _P]),
    "convrot_combine_rows": (_I, [_P, _P, _P, _I, _I64, _I64, _I64, _P, _P]),
    "convrot_gather_rows": (_I, [_P, _P, _I64, _P, _I64, _I64, _P, _P, _P]),
    "convrot_i8_gemm_i32": (_I, [_P, _P, _I, _I64, _I64, _I64, _I64, _P, _P]),
    "convrot_i8_gemm_bf16": (_I, [_P, _P, _P, _P, _I, _I64, _I64, _I64, _I64, _P, _P]),
    "convrot_i8_gemm_swiglu": (_I, [_P, _P, _P, _P, _I, _I64, _I64, _I64, _I64, _P, _P]),
    "convrot_swiglu_rq_sync_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "convrot_i8_gemm_swiglu_rq": (_I, [_P, _P, _P, _P, _I, _I64, _I64, _I64, _I64, _I, _P, _P,
                                       _P, ctypes.c_size_t, _P]),
    "convrot_i8_gemm_scatter": (_I, [_P, _P, _P, _P, _I, _P, _P, _I64, _I64, _I64, _I64, _P, _I64,
                                     _P]),
    "convrot_f32_to_bf16": (_I, [_P, _I64, _P, _P]),
    "convrot_linear_workspace_size": (_SZ, [_I64, _I64]),
    "w8a8_convrot_linear": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _P, _P, _SZ, _P]),
    "w8a8_convrot_linear_noalloc": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _P, _P]),
    "moe_workspace_layout": (_I, [_I64, _I64, _I64, _I, _I64, ctypes.POINTER(MoeLayout)]),
    "moe_workspace_size": (_SZ, [_I64, _I64, _I64, _I, _I64]),
    "moe_expert_choice_forward": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I64, _I, _I,
                                       _P, _P, _SZ, _P]),
    "convrot_lowbit_weight_bytes": (_I64, [_I64, _I64, _I]),
    "convrot_quantize_weights_lowbit": (_I, [_P, _I64, _I64, _I, _I, _P, _P, _P]),
    "convrot_lowbit_gemm": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _P, _P]),
    "lowbit_convrot_linear": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _I, _P, _P, _SZ, _P]),
    "moe_expert_choice_forward_lowbit": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I64,
                                              _I, _I, _I, _P, _P, _SZ, _P]),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libconvrot.so and declares every C signature. Raises if missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with `python -m w8a8_rotated_int8_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def lib() -> ctypes.CDLL:
    return _lib if _lib is not None else load_library()


def status_string(status: int) -> str:
    return lib().convrot_status_string(status).decode()


def _check(rc: int, where: str):
    if rc != CONVROT_OK:
        raise ConvrotError(rc, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None, like=None):
    """The given stream, else the current stream of `like`'s device (else of
    the current device)."""
    if stream is None:
        stream = torch.cuda.current_stream(None if like is None else like.device)
    return ctypes.c_void_p(stream.cuda_stream)


def _invoke(t, name, *args, stream=None):
    """Calls the C entry `name` with `t`'s device current (the library works on
    the current device) and that device's current stream (or `stream`) as the
    last argument; raises on a non-OK status."""
    with torch.cuda.device(t.device):
        rc = getattr(lib(), name)(*args, _stream(stream, t))
    _check(rc, name)


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------- diagnostics --
def convrot_device_check():
    _check(lib().convrot_device_check(), "convrot_device_check")


def convrot_check_device_error(stream=None) -> int:
    """Synchronises and returns the device error bits (0 = none); clears them."""
    flags = ctypes.c_uint(0)
    rc = lib().convrot_check_device_error(_stream(stream), ctypes.byref(flags))
    if rc not in (CONVROT_OK, CONVROT_ERR_TIMEOUT):
        raise ConvrotError(rc, "convrot_check_device_error")
    return int(flags.value)


def convrot_wait_selftest(limit_ns: int, stream=None) -> int:
    """Runs the bounded-wait self-test; returns 0 when the wait gave up."""
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _invoke(res, "convrot_wait_selftest", limit_ns, _p(res), stream=stream)
    return int(res.item())


def convrot_count_wait_selftest(limit_ns: int, stream=None) -> int:
    """Runs the bounded cross-CTA counter wait on a counter nothing raises;
    returns 0 when the wait gave up."""
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    words = torch.empty((2,), dtype=torch.int32, device="cuda")
    _invoke(res, "convrot_count_wait_selftest", limit_ns, _p(words), _p(res), stream=stream)
    return int(res.item())


def convrot_swiglu_rq_units(tiles: int, n_blocks: int, capacity: int) -> int:
    """Host rule: co-resident units the requantising GEMM runs on (0 = it
    cannot run, the two-step path is used instead)."""
    return int(lib().convrot_swiglu_rq_units(tiles, n_blocks, capacity))


# ------------------------------------------------------------------ stages --
def convrot_rotquant(x, group, q=None, scale=None, stream=None):
    """Rotate rows of x ([rows, K] bf16 or fp32) in groups of `group`, then
    quantise per row. Returns (codes int8 [rows, K], scales fp32 [rows])."""
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x must be bf16 or fp32")
    _need(x, x.dtype, "x")
    rows, k = x.shape
    q = torch.empty((rows, k), dtype=torch.int8, device=x.device) if q is None else q
    scale = torch.empty((rows,), dtype=torch.float32, device=x.device) if scale is None else scale
    dt = DTYPE_BF16 if x.dtype == torch.bfloat16 else DTYPE_F32
    _invoke(x, "convrot_rotquant", _p(x), dt, rows, k, group, _p(q), _p(scale), stream=stream)
    return q, scale


def convrot_quantize_weights(w, group, stream=None):
    """Offline quantisation of bf16 weight rows; [..., K] -> (codes, scales [...])."""
    _need(w, torch.bfloat16, "w")
    k = w.shape[-1]
    rows = w.numel() // k
    q = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    s = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    _invoke(w, "convrot_quantize_weights", _p(w), rows, k, group, _p(q), _p(s), stream=stream)
    return q, s


def tiled_weight_bytes(n_mats, rows, k) -> int:
    return int(lib().convrot_tiled_weight_bytes(n_mats, rows, k))


class TiledWeights:
    """Codes in the tiled weight format plus their per-row scales."""

    def __init__(self, data, scale, n_mats, rows, k):
        self.data, self.scale, self.n_mats, self.rows, self.k = data, scale, n_mats, rows, k


def convrot_quantize_weights_tiled(w, group, n_mats, stream=None):
    """Quantise bf16 rows (n_mats matrices stacked along rows) into the tiled
    weight format. Returns TiledWeights(data uint8-bytes as int8, scale)."""
    _need(w, torch.bfloat16, "w")
    k = w.shape[-1]
    total = w.numel() // k
    if total % n_mats:
        raise ValueError("rows must split evenly into n_mats matrices")
    rows = total // n_mats
    data = torch.empty((tiled_weight_bytes(n_mats, rows, k),), dtype=torch.int8, device=w.device)
    scale = torch.empty((total,), dtype=torch.float32, device=w.device)
    _invoke(w, "convrot_quantize_weights_tiled", _p(w),
            n_mats, rows, k, group, _p(data), _p(scale), stream=stream)
    return TiledWeights(data, scale, n_mats, rows, k)


def untile(tw: TiledWeights):
    """Row-major [n_mats * rows, K] view of tiled codes (a copy; for checks)."""
    kb = -(-tw.k // 128)
    rb = -(-tw.rows // 128)
    t = tw.data.view(tw.n_mats, rb, kb, 128, 128).permute(0, 1, 3, 2, 4)
    t = t.reshape(tw.n_mats, rb * 128, kb * 128)[:, :tw.rows, :tw.k]
    return t.reshape(tw.n_mats * tw.rows, tw.k)


def convrot_router_softmax(logits, stream=None):
    """[T, E] bf16 logits -> transposed scores [E, T] fp32."""
    _need(logits, torch.bfloat16, "logits")
    t, e = logits.shape
    s_t = torch.empty((e, t), dtype=torch.float32, device=logits.device)
    _invoke(logits, "convrot_router_softmax", _p(logits), t, e, _p(s_t), stream=stream)
    return s_t


def convrot_topc(s_t, c, with_slot=False, stream=None):
    """[E, T] fp32 scores -> (idx int32 [E, C], w fp32 [E, C]) and, with
    with_slot, slot int32 [E, T] (position of each token per expert or -1)."""
    _need(s_t, torch.float32, "s_t")
    e, t = s_t.shape
    idx = torch.empty((e, c), dtype=torch.int32, device=s_t.device)
    w = torch.empty((e, c), dtype=torch.float32, device=s_t.device)
    slot = torch.empty((e, t), dtype=torch.int32, device=s_t.device) if with_slot else None
    _invoke(s_t, "convrot_topc", _p(s_t), t, e, c, _p(idx), _p(w), _p(slot), stream=stream)
    return (idx, w, slot) if with_slot else (idx, w)


def convrot_combine_rows(z, s_t, slot, c, stream=None):
    """z [E*C, d] bf16 expert outputs, s_t [E, T] fp32 router scores, slot
    [E, T] -> y [T, d] bf16 (per token, the fp32 sum of s_t * z over its
    experts in ascending expert order)."""
    _need(z, torch.bfloat16, "z")
    _need(s_t, torch.float32, "s_t")
    _need(slot, torch.int32, "slot")
    e, t = slot.shape
    d = z.shape[-1]
    y = torch.empty((t, d), dtype=torch.bfloat16, device=slot.device)
    _invoke(z, "convrot_combine_rows", _p(z), _p(s_t), _p(slot), e, t, c, d, _p(y), stream=stream)
    return y


def convrot_gather_rows(src, s_src, idx, stream=None):
    _need(src, torch.int8, "src")
    _need(s_src, torch.float32, "s_src")
    _need(idx, torch.int32, "idx")
    n_src, k = src.shape
    n = idx.numel()
    dst = torch.empty((n, k), dtype=torch.int8, device=src.device)
    s_dst = torch.empty((n,), dtype=torch.float32, device=src.device)
    _invoke(src, "convrot_gather_rows", _p(src),
            _p(s_src), n_src, _p(idx), n, k, _p(dst), _p(s_dst), stream=stream)
    return dst, s_dst


def _gemm_dims(a, b, swiglu=False):
    """(G, M, N, K, b pointer tensor, layout). b is a row-major [G, N, K]
    (or [N, K]) int8 tensor or TiledWeights."""
    _need(a, torch.int8, "a")
    if a.dim() == 2:
        a = a[None]
    g, m, k = a.shape
    if isinstance(b, TiledWeights):
        per = 2 if swiglu else 1
        if b.n_mats != g * per or b.k != k:
            raise ValueError("tiled weights do not match a [G,M,K]")
        return g, m, b.rows * per, k, b.data, LAYOUT_TILES
    _need(b, torch.int8, "b")
    if b.dim() == 2:
        b = b[None]
    gb, n, kb = b.shape
    if gb != g or kb != k:
        raise ValueError("a [G,M,K] and b [G,N,K] disagree")
    return g, m, n, k, b, LAYOUT_ROWS


def convrot_i8_gemm_i32(a, b, stream=None):
    """Exact int32 acc[g, m, n] = sum_k a[g, m, k] b[g, n, k]."""
    g, m, n, k, bt, lay = _gemm_dims(a, b)
    d = torch.empty((g, m, n), dtype=torch.int32, device=a.device)
    _invoke(a, "convrot_i8_gemm_i32", _p(a), _p(bt), lay, g, m, n, k, _p(d), stream=stream)
    return d if a.dim() == 3 else d[0]


def convrot_i8_gemm_bf16(a, s_a, b, s_b, stream=None):
    g, m, n, k, bt, lay = _gemm_dims(a, b)
    _need(s_a, torch.float32, "s_a")
    _need(s_b, torch.float32, "s_b")
    y = torch.empty((g, m, n), dtype=torch.bfloat16, device=a.device)
    _invoke(a, "convrot_i8_gemm_bf16", _p(a),
            _p(s_a), _p(bt), _p(s_b), lay, g, m, n, k, _p(y), stream=stream)
    return y if a.dim() == 3 else y[0]


def convrot_i8_gemm_swiglu(a, s_a, b, s_b, stream=None):
    """b = [G, 2F, K] (gate rows then up rows) or tiled (2G matrices of F
    rows) -> h [G, M, F] fp32."""
    g, m, n2, k, bt, lay = _gemm_dims(a, b, swiglu=True)
    _need(s_a, torch.float32, "s_a")
    _need(s_b, torch.float32, "s_b")
    f = n2 // 2
    h = torch.empty((g, m, f), dtype=torch.float32, device=a.device)
    _invoke(a, "convrot_i8_gemm_swiglu", _p(a),
            _p(s_a), _p(bt), _p(s_b), lay, g, m, f, k, _p(h), stream=stream)
    return h if a.dim() == 3 else h[0]


def convrot_i8_gemm_swiglu_rq(a, s_a, b, s_b, g_h=64, stream=None):
    """SwiGLU, then h rotated in groups of g_h and requantised per row, all in
    the GEMM epilogue -> (h_q [G, M, F] int8, s_h [G, M] fp32)."""
    g, m, n2, k, bt, lay = _gemm_dims(a, b, swiglu=True)
    _need(s_a, torch.float32, "s_a")
    _need(s_b, torch.float32, "s_b")
    f = n2 // 2
    h_q = torch.empty((g, m, f), dtype=torch.int8, device=a.device)
    s_h = torch.empty((g, m), dtype=torch.float32, device=a.device)
    nbytes = lib().convrot_swiglu_rq_sync_bytes(g, m)
    sync = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=a.device)
    _invoke(a, "convrot_i8_gemm_swiglu_rq", _p(a), _p(s_a), _p(bt), _p(s_b), lay, g, m, f, k,
            g_h, _p(h_q), _p(s_h), _p(sync), nbytes, stream=stream)
    return (h_q, s_h) if a.dim() == 3 else (h_q[0], s_h[0])


def convrot_i8_gemm_scatter(a, s_a, b, s_b, idx, w, out32, stream=None):
    """out32[idx[g, m], n] += w[g, m] * dequant(acc)[g, m, n] (in place)."""
    g, m, n, k, bt, lay = _gemm_dims(a, b)
    for t, nm in ((s_a, "s_a"), (s_b, "s_b"), (w, "w"), (out32, "out32")):
        _need(t, torch.float32, nm)
    _need(idx, torch.int32, "idx")
    _invoke(a, "convrot_i8_gemm_scatter", _p(a), _p(s_a), _p(bt), _p(s_b), lay, _p(idx),
            _p(w), g, m, n, k, _p(out32), out32.shape[0], stream=stream)
    return out32


def convrot_f32_to_bf16(x, stream=None):
    _need(x, torch.float32, "x")
    y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _invoke(x, "convrot_f32_to_bf16", _p(x), x.numel(), _p(y), stream=stream)
    return y


# ---------------------------------------------------------------- linears --
def convrot_linear_workspace_size(m, k) -> int:
    return int(lib().convrot_linear_workspace_size(m, k))


def w8a8_convrot_linear(x, w_q, w_scale, group, y=None, workspace=None, stream=None):
    """Y[M, N] bf16 = W8A8 ConvRot linear of x [M, K] bf16 with rotated codes w_q [N, K]."""
    _need(x, torch.bfloat16, "x")
    _need(w_q, torch.int8, "w_q")
    _need(w_scale, torch.float32, "w_scale")
    m, k = x.shape
    n = w_q.shape[0]
    ws_bytes = convrot_linear_workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _invoke(x, "w8a8_convrot_linear", _p(x), m, k, _p(w_q), _p(w_scale), n, group, _p(y),
            _p(workspace), workspace.numel(), stream=stream)
    return y


def w8a8_convrot_linear_noalloc(x, w_q, w_scale, group, y=None, stream=None):
    """The W8A8 ConvRot linear with the library's static scratch instead of a
    workspace, for callers that cannot give the library device memory.
    M * K <= 8,388,608 and M <= 16,384; calls sharing the scratch must be
    ordered on one stream."""
    _need(x, torch.bfloat16, "x")
    _need(w_q, torch.int8, "w_q")
    _need(w_scale, torch.float32, "w_scale")
    m, k = x.shape
    n = w_q.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _invoke(x, "w8a8_convrot_linear_noalloc", _p(x),
            m, k, _p(w_q), _p(w_scale), n, group, _p(y), stream=stream)
    return y


# -------------------------------------------------------------- MoE block --
def moe_workspace_layout(t, d, f, e, c) -> dict:
    lay = MoeLayout()
    _check(lib().moe_workspace_layout(t, d, f, e, c, ctypes.byref(lay)), "moe_workspace_layout")
    return {name: int(getattr(lay, name)) for name, _ in MoeLayout._fields_}


def moe_workspace_size(t, d, f, e, c) -> int:
    return int(lib().moe_workspace_size(t, d, f, e, c))


def quantize_moe_weights(wgu, wd, g_gu=256, g_d=64, stream=None):
    """Offline: bf16 wgu [E, 2f, d] and wd [E, d, f] -> tiled codes + scales."""
    e, two_f, d = wgu.shape
    gu = convrot_quantize_weights_tiled(wgu.reshape(e * two_f, d), g_gu, 2 * e, stream=stream)
    dn = convrot_quantize_weights_tiled(wd.reshape(-1, wd.shape[-1]), g_d, e, stream=stream)
    return gu, dn


def moe_expert_choice_forward(x, logits, w_gu, w_d, c, g_gu=256, g_d=64, y=None,
                              workspace=None, stream=None):
    """Expert-choice W8A8 ConvRot MoE block. x [T, d] bf16, logits [T, E] bf16,
    w_gu / w_d = TiledWeights from quantize_moe_weights -> y [T, d] bf16."""
    _need(x, torch.bfloat16, "x")
    _need(logits, torch.bfloat16, "logits")
    t, d = x.shape
    e = logits.shape[1]
    f = w_gu.rows
    if w_gu.n_mats != 2 * e or w_gu.k != d or w_d.n_mats != e or w_d.rows != d or w_d.k != f:
        raise ValueError("weights do not match x / logits")
    s_gu, s_d = w_gu.scale, w_d.scale
    w_gu, w_d = w_gu.data, w_d.data
    size = moe_workspace_size(t, d, f, e, c)
    if workspace is None:
        workspace = torch.empty((max(size, 16),), dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty((t, d), dtype=torch.bfloat16, device=x.device)
    _invoke(x, "moe_expert_choice_forward", _p(x), _p(logits), _p(w_gu), _p(s_gu), _p(w_d),
            _p(s_d), t, d, f, e, c, g_gu, g_d, _p(y), _p(workspace), workspace.numel(),
            stream=stream)
    return y


def moe_stage_views(workspace, t, d, f, e, c) -> dict:
    """Typed views of every intermediate the MoE call leaves in its workspace."""
    lay = moe_workspace_layout(t, d, f, e, c)

    def view(name, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return workspace[lay[name]:lay[name] + nbytes].view(dtype).view(shape)

    return {
        "x_q": view("x_q", torch.int8, (t, d)),
        "s_x": view("s_x", torch.float32, (t,)),
        "s_t": view("s_t", torch.float32, (e, t)),
        "idx": view("idx", torch.int32, (e, c)),
        "w": view("w", torch.float32, (e, c)),
        "x_g": view("x_g", torch.int8, (e, c, d)),
        "s_g": view("s_g", torch.float32, (e, c)),
        "h": view("h", torch.float32, (e, c, f)),
        "h_q": view("h_q", torch.int8, (e, c, f)),
        "s_h": view("s_h", torch.float32, (e, c)),
        "slot": view("slot", torch.int32, (e, t)),
        "z": view("z", torch.bfloat16, (e, c, d)),
    }


# ------------------------------------------------------- W4A8 / W6A8 --------
CONVROT_LOWBIT_F32, CONVROT_LOWBIT_BF16, CONVROT_LOWBIT_SWIGLU = 0, 1, 2


def lowbit_weight_bytes(rows, k, bits) -> int:
    return int(lib().convrot_lowbit_weight_bytes(rows, k, bits))


class LowbitWeights:
    """Weights in the packed b-bit format (uint8 bytes) plus their FP32 row
    scales; `rows` rows of each of `n_mats` matrices, K columns."""

    def __init__(self, data, scale, n_mats, rows, k, bits):
        self.data, self.scale = data, scale
        self.n_mats, self.rows, self.k, self.bits = n_mats, rows, k, bits


def convrot_quantize_weights_lowbit(w, group, bits, n_mats=1, stream=None):
    """Offline: bf16 weight rows [..., K] (n_mats matrices stacked along the
    rows, each a multiple of 128 rows) -> LowbitWeights."""
    _need(w, torch.bfloat16, "w")
    k = w.shape[-1]
    total = w.numel() // k
    if total % n_mats:
        raise ValueError("rows must split evenly into n_mats matrices")
    nbytes = lowbit_weight_bytes(total, k, bits)
    if nbytes < 0:
        raise ValueError("rows must be a multiple of 128 and K of 64; bits 4 or 6")
    data = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=w.device)
    scale = torch.empty((total,), dtype=torch.float32, device=w.device)
    _invoke(w, "convrot_quantize_weights_lowbit", _p(w), total, k, group, bits, _p(data),
            _p(scale), stream=stream)
    return LowbitWeights(data, scale, n_mats, total // n_mats, k, bits)


def convrot_lowbit_gemm(a, s_a, w: LowbitWeights, epilogue=CONVROT_LOWBIT_BF16, tile_tokens=0,
                        out=None, stream=None):
    """Grouped low-bit GEMM: a [G, M, K] int8 codes (s_a [G, M] fp32) against
    the G matrices of w. epilogue F32 -> acc [G, M, N] fp32; BF16 -> y bf16;
    SWIGLU -> h [G, M, N/2] fp32."""
    _need(a, torch.int8, "a")
    if s_a is not None:
        _need(s_a, torch.float32, "s_a")
    g, m, k = a.shape
    if w.n_mats != g or w.k != k:
        raise ValueError("weights do not match a")
    n = w.rows
    if epilogue == CONVROT_LOWBIT_BF16:
        shape, dtype = (g, m, n), torch.bfloat16
    elif epilogue == CONVROT_LOWBIT_SWIGLU:
        shape, dtype = (g, m, n // 2), torch.float32
    else:
        shape, dtype = (g, m, n), torch.float32
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=a.device)
    elif out.numel() != g * m * (n // 2 if epilogue == CONVROT_LOWBIT_SWIGLU else n):
        raise ValueError("out has the wrong size")
    else:
        _need(out, dtype, "out")
    _invoke(a, "convrot_lowbit_gemm", _p(a), _p(s_a), _p(w.data), _p(w.scale), g, m, n, k,
            w.bits, epilogue, tile_tokens, _p(out), stream=stream)
    return out


def lowbit_convrot_linear(x, w: LowbitWeights, group, y=None, workspace=None, stream=None):
    """Y[M, N] bf16 = WbA8 ConvRot linear of x [M, K] bf16 against b-bit weights."""
    _need(x, torch.bfloat16, "x")
    m, k = x.shape
    if w.n_mats != 1 or w.k != k:
        raise ValueError("weights do not match x")
    n = w.rows
    ws_bytes = convrot_linear_workspace_size(m, k)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _invoke(x, "lowbit_convrot_linear", _p(x), m, k, _p(w.data), _p(w.scale), n, group, w.bits,
            _p(y), _p(workspace), workspace.numel(), stream=stream)
    return y


def quantize_moe_weights_lowbit(wgu, wd, bits, g_gu=256, g_d=64, stream=None):
    """Offline: bf16 wgu [E, 2f, d] and wd [E, d, f] -> LowbitWeights (E matrices each)."""
    e = wgu.shape[0]
    gu = convrot_quantize_weights_lowbit(wgu.reshape(-1, wgu.shape[-1]), g_gu, bits, e,
                                         stream=stream)
    dn = convrot_quantize_weights_lowbit(wd.reshape(-1, wd.shape[-1]), g_d, bits, e,
                                         stream=stream)
    return gu, dn


def moe_expert_choice_forward_lowbit(x, logits, w_gu: LowbitWeights, w_d: LowbitWeights, c,
                                     g_gu=256, g_d=64, y=None, workspace=None, stream=None):
    """The expert-choice MoE block with b-bit expert weights (from
    quantize_moe_weights_lowbit); x [T, d] bf16, logits [T, E] bf16 -> y."""
    _need(x, torch.bfloat16, "x")
    _need(logits, torch.bfloat16, "logits")
    t, d = x.shape
    e = logits.shape[1]
    f = w_gu.rows // 2
    if (w_gu.n_mats != e or w_gu.k != d or w_d.n_mats != e or w_d.rows != d or w_d.k != f
            or w_gu.bits != w_d.bits):
        raise ValueError("weights do not match x / logits")
    size = moe_workspace_size(t, d, f, e, c)
    if workspace is None:
        workspace = torch.empty((max(size, 16),), dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty((t, d), dtype=torch.bfloat16, device=x.device)
    _invoke(x, "moe_expert_choice_forward_lowbit", _p(x), _p(logits), _p(w_gu.data),
            _p(w_gu.scale), _p(w_d.data), _p(w_d.scale), t, d, f, e, c, g_gu, g_d, w_gu.bits,
            _p(y), _p(workspace), workspace.numel(), stream=stream)
    return y
