"""The no-allocation W8A8 ConvRot linear against the workspace entry point.

w8a8_convrot_linear_noalloc serves callers that cannot give the library
device memory (a host program holding only its tensors and no device
allocator, a serving loop where cudaMalloc/cudaFree would synchronise the
device, a fixed memory budget). Its scratch is one static device array in the
library. This file runs last so that a failure here never hides another test.
"""

import ctypes

import pytest
import torch

from synthetic import LINEAR_CONFIGS, linear_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import w8a8_rotated_int8_b200 as lib_mod
    lib_mod.load_library()
    lib_mod.convrot_device_check()
    return lib_mod


def _quantised(W, name):
    cfg = LINEAR_CONFIGS[name]
    x, w = linear_inputs(cfg)
    w_q, s_w = W.convrot_quantize_weights(w.cuda(), cfg.group)
    return cfg, x.cuda(), w_q, s_w


def test_noalloc_matches_workspace_entry_two_calls_in_a_row(W):
    # two different problems back to back through the same static scratch;
    # the first fills it to its limit (4096 x 2048 codes = 8,388,608 bytes)
    runs = [_quantised(W, "gateup_4096x3072x2048"), _quantised(W, "down_4096x2048x1536")]
    outs = []
    for cfg, x, w_q, s_w in runs:
        outs.append(W.w8a8_convrot_linear_noalloc(x, w_q, s_w, cfg.group))
    torch.cuda.synchronize()
    for (cfg, x, w_q, s_w), y in zip(runs, outs):
        ref = W.w8a8_convrot_linear(x, w_q, s_w, cfg.group)
        torch.cuda.synchronize()
        # both paths run the same kernels on the same codes: bit-identical
        assert torch.equal(y, ref), cfg.name
    assert W.convrot_check_device_error() == 0


def test_noalloc_small_and_ragged_shapes(W):
    """A single-CTA GEMM of 64 rows (its rows in TMEM lanes 64..127) and a row
    count that is not a multiple of 128, each twice in a row through the
    shared scratch, bit-identical to the workspace entry point."""
    cfg, x, w_q, s_w = _quantised(W, "linear_64x256x256")
    gen = torch.Generator().manual_seed(9)
    x2 = torch.randn(200, 512, generator=gen).to(torch.bfloat16).cuda()
    w2 = (torch.randn(320, 512, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    w2_q, s2_w = W.convrot_quantize_weights(w2, 64)
    cases = [(x, w_q, s_w, cfg.group), (x2, w2_q, s2_w, 64)]
    for _ in range(2):
        for xx, wq, sw, g in cases:
            y = W.w8a8_convrot_linear_noalloc(xx, wq, sw, g)
            ref = W.w8a8_convrot_linear(xx, wq, sw, g)
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
    assert W.convrot_check_device_error() == 0


def test_noalloc_rejects_problems_beyond_the_static_scratch(W):
    from w8a8_rotated_int8_b200 import binding
    lib = binding.lib()
    dev = ctypes.c_void_p(torch.empty(16, device="cuda").data_ptr())
    too_many_codes = lib.w8a8_convrot_linear_noalloc(dev, 4097, 2048, dev, dev, 256, 256, dev, None)
    too_many_rows = lib.w8a8_convrot_linear_noalloc(dev, 16385, 256, dev, dev, 256, 256, dev, None)
    assert too_many_codes == binding.CONVROT_ERR_WORKSPACE_TOO_SMALL
    assert too_many_rows == binding.CONVROT_ERR_WORKSPACE_TOO_SMALL
    # an invalid K is reported as such even when the problem is also too big
    bad_k = lib.w8a8_convrot_linear_noalloc(dev, 20000, 17, dev, dev, 256, 1, dev, None)
    assert bad_k == binding.CONVROT_ERR_INVALID_ARG
    # host memory is not the current device's
    host = torch.empty(64 * 256, dtype=torch.bfloat16).pin_memory()
    w_q = torch.zeros(256, 256, dtype=torch.int8, device="cuda")
    s_w = torch.ones(256, device="cuda")
    y = torch.empty(64, 256, dtype=torch.bfloat16, device="cuda")
    rc = lib.w8a8_convrot_linear_noalloc(ctypes.c_void_p(host.data_ptr()), 64, 256,
                                         ctypes.c_void_p(w_q.data_ptr()),
                                         ctypes.c_void_p(s_w.data_ptr()), 256, 256,
                                         ctypes.c_void_p(y.data_ptr()), None)
    assert rc == binding.CONVROT_ERR_INVALID_ARG
    assert W.convrot_check_device_error() == 0
