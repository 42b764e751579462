"""The C-ABI library loads without a GPU, exports every declared symbol, and
rejects bad arguments on the host before touching the device (no GPU)."""

import ctypes
import os
import re

import pytest

from w8a8_rotated_int8_b200 import binding
from w8a8_rotated_int8_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("convrot_quantize_weights", "w8a8_convrot_linear",
                     "moe_expert_choice_forward", "convrot_rotquant", "convrot_topc",
                     "convrot_i8_gemm_i32"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(binding._SIGNATURES) == set(declared_functions())


def test_abi_version_and_strings(lib):
    assert lib.convrot_abi_version() == 3
    for code in range(7):
        assert binding.status_string(code)
    assert binding.status_string(99) == "unknown status"


def test_argument_checks_need_no_gpu(lib):
    al = ctypes.c_void_p(4096)       # 16-byte aligned placeholder, never dereferenced
    mis = ctypes.c_void_p(4096 + 8)
    INVALID, MISALIGNED = binding.CONVROT_ERR_INVALID_ARG, binding.CONVROT_ERR_MISALIGNED
    # unsupported rotation group / K not a multiple of the group / K % 16
    assert lib.convrot_rotquant(al, 0, 4, 256, 128, al, al, None) == INVALID
    assert lib.convrot_rotquant(al, 0, 4, 96, 64, al, al, None) == INVALID
    assert lib.convrot_rotquant(al, 0, 4, 40, 4, al, al, None) == INVALID
    assert lib.convrot_rotquant(al, 7, 4, 256, 256, al, al, None) == INVALID
    assert lib.convrot_rotquant(mis, 0, 4, 256, 256, al, al, None) == MISALIGNED
    # top-C capacity beyond T
    assert lib.convrot_topc(al, 10, 4, 11, al, al, None, None) == INVALID
    # GEMM: K not a multiple of 16, N not a multiple of 16, int32 overflow bound
    assert lib.convrot_i8_gemm_i32(al, al, 0, 1, 8, 16, 40, al, None) == INVALID
    assert lib.convrot_i8_gemm_i32(al, al, 0, 1, 8, 24, 64, al, None) == INVALID
    assert lib.convrot_i8_gemm_i32(al, al, 0, 1, 8, 16, 1 << 20, al, None) == INVALID
    assert lib.convrot_i8_gemm_i32(al, al, 2, 1, 8, 16, 64, al, None) == INVALID  # bad layout
    # requantising SwiGLU GEMM: a group that does not fit one thread (256), a group that is not
    # a power of four, F not a multiple of the group, a misaligned output, a scratch too small
    rq = lib.convrot_i8_gemm_swiglu_rq
    big = 1 << 20
    assert rq(al, al, al, al, 1, 2, 64, 256, 256, 256, al, al, al, big, None) == INVALID
    assert rq(al, al, al, al, 1, 2, 64, 256, 256, 8, al, al, al, big, None) == INVALID
    assert rq(al, al, al, al, 1, 2, 64, 80, 256, 64, al, al, al, big, None) == INVALID
    assert rq(al, al, al, al, 1, 2, 64, 256, 256, 64, mis, al, al, big, None) == MISALIGNED
    assert (rq(al, al, al, al, 1, 2, 64, 256, 256, 64, al, al, al, 64, None)
            == binding.CONVROT_ERR_WORKSPACE_TOO_SMALL)
    # its scratch: the row maxima (256-byte aligned), then an arrival counter per 128-row slab
    # (one spare slab per group), the abort word and a published-tile count per group
    assert lib.convrot_swiglu_rq_sync_bytes(64, 256) == 64 * 256 * 4 + (64 * 3 + 1 + 64) * 4
    assert lib.convrot_swiglu_rq_sync_bytes(5, 40) == 1024 + (5 * 2 + 1 + 5) * 4
    # tiled weight sizes: 128-row blocks x 128-byte K tiles of 16 KB
    assert lib.convrot_tiled_weight_bytes(2, 300, 200) == 2 * 3 * 2 * 16384
    assert lib.convrot_tiled_weight_bytes(128, 1536, 2048) == 128 * 12 * 16 * 16384
    # MoE: C > T, bad group, d not a multiple of g_gu, workspace too small
    args = [al] * 6
    assert lib.moe_expert_choice_forward(*args, 8, 256, 64, 4, 9, 256, 64, al, al, 1 << 30, None) == INVALID
    assert lib.moe_expert_choice_forward(*args, 8, 256, 64, 4, 2, 32, 64, al, al, 1 << 30, None) == INVALID
    assert lib.moe_expert_choice_forward(*args, 8, 320, 64, 4, 2, 256, 64, al, al, 1 << 30, None) == INVALID
    assert (lib.moe_expert_choice_forward(*args, 8, 256, 64, 4, 2, 256, 64, al, al, 16, None)
            == binding.CONVROT_ERR_WORKSPACE_TOO_SMALL)


def test_no_device_is_reported_not_crashed(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.convrot_device_check() == binding.CONVROT_ERR_UNSUPPORTED_DEVICE


def test_workspace_layout_is_disjoint_and_aligned(lib):
    lay = binding.moe_workspace_layout(8192, 2048, 1536, 64, 256)
    names = [n for n in lay if n != "total"]
    offs = sorted(lay[n] for n in names)
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == len(offs)
    assert lay["total"] >= lay["z"] + 64 * 256 * 2048 * 2


def test_requantising_gemm_plan_falls_back_when_too_few_ctas_fit(lib):
    """The host rule for the requantising gate/up GEMM: its tiles of one row
    block wait for one another, so it runs only on a capacity that holds a
    whole row block's tiles at once; with less (a share of the SMs) the plan
    is 0 and the library takes the two-step path instead of launching waits
    that could not end."""
    units = binding.convrot_swiglu_rq_units
    # T=8192: 64 experts x 1 pair m-block x 12 n-blocks = 768 tiles, 74 pairs fit
    assert units(768, 12, 74) == 72            # six whole row blocks per wave
    assert units(768, 12, 11) == 0             # one row block cannot meet: fall back
    assert units(768, 12, 12) == 12
    assert units(30, 12, 74) == 30             # every tile fits at once
    assert units(0, 12, 74) == 0
    assert units(-1, 12, 74) == -1


def test_lowbit_argument_checks_need_no_gpu(lib):
    """W4A8 / W6A8 entry points: format sizes and host-side rejections."""
    al = ctypes.c_void_p(4096)
    mis = ctypes.c_void_p(4096 + 8)
    INVALID, MISALIGNED = binding.CONVROT_ERR_INVALID_ARG, binding.CONVROT_ERR_MISALIGNED
    # tiles of 128 rows x 64 codes: 2 planes + 512 scale bytes (4-bit), 3 planes (6-bit)
    assert lib.convrot_lowbit_weight_bytes(128, 64, 4) == 4608
    assert lib.convrot_lowbit_weight_bytes(6144, 2048, 6) == 48 * 32 * 6656
    assert lib.convrot_lowbit_weight_bytes(128, 64, 8) == -1
    assert lib.convrot_lowbit_weight_bytes(200, 64, 4) == -1
    assert lib.convrot_lowbit_weight_bytes(128, 96, 4) == -1
    q = lib.convrot_quantize_weights_lowbit
    assert q(al, 128, 256, 256, 5, al, al, None) == INVALID       # bits
    assert q(al, 100, 256, 256, 4, al, al, None) == INVALID       # rows % 128
    assert q(al, 128, 320, 256, 4, al, al, None) == INVALID       # K % group
    assert q(al, 128, 96, 16, 4, al, al, None) == INVALID         # K % 64
    assert q(al, 128, 256, 128, 4, al, al, None) == INVALID       # group not a power of four
    assert q(mis, 128, 256, 256, 4, al, al, None) == MISALIGNED
    g = lib.convrot_lowbit_gemm
    assert g(al, al, al, al, 1, 64, 128, 256, 4, 1, 0, al, None) == INVALID   # N % 256
    assert g(al, al, al, al, 1, 64, 256, 96, 4, 1, 0, al, None) == INVALID    # K % 64
    assert g(al, al, al, al, 1, 64, 256, 256, 4, 3, 0, al, None) == INVALID   # epilogue
    assert g(al, al, al, al, 1, 64, 256, 256, 4, 1, 24, al, None) == INVALID  # tile tokens
    assert g(al, al, al, al, 1, 64, 256, 256, 4, 1, 144, al, None) == INVALID
    assert g(mis, al, al, al, 1, 64, 256, 256, 4, 1, 0, al, None) == MISALIGNED
    assert g(al, al, al, mis, 1, 64, 256, 256, 4, 1, 0, al, None) == MISALIGNED  # row scales
    lin = lib.lowbit_convrot_linear
    assert lin(al, 64, 256, al, al, 256, 256, 4, al, al, 16, None) == \
        binding.CONVROT_ERR_WORKSPACE_TOO_SMALL
    assert lin(al, 64, 256, al, al, 384, 256, 4, al, al, 1 << 20, None) == INVALID
    assert lin(al, 64, 256, al, mis, 256, 256, 4, al, al, 1 << 20, None) == MISALIGNED
    m = lib.moe_expert_choice_forward_lowbit
    args = [al] * 6
    assert m(*args, 8, 256, 192, 4, 2, 256, 64, 4, al, al, 1 << 30, None) == INVALID  # f % 128
    assert m(*args, 8, 320, 128, 4, 2, 64, 64, 4, al, al, 1 << 30, None) == INVALID   # d % 256
    assert m(*args, 8, 256, 128, 4, 2, 256, 64, 5, al, al, 1 << 30, None) == INVALID  # bits
    assert (m(*args, 8, 256, 128, 4, 2, 256, 64, 4, al, al, 16, None)
            == binding.CONVROT_ERR_WORKSPACE_TOO_SMALL)
