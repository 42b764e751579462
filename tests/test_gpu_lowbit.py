"""GPU parity of the W4A8 / W6A8 path through the C ABI against the oracle.

Source: "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were
made" (6-bit / 4-bit weights in the rotated basis, an FP8 scale per group of
16, 8-bit activations); readings in oracle/lowbit_oracle.py.

Bar: the offline quantiser bit-exact (codes, E4M3 group scales, FP32 row
scales); the GEMM's accumulator within the fp32 summation bound
K * 2^-23 * sum_k |x * sigma * q| of the exact sum (the operands are exact
fp16 and every product exact, so only the order of the fp32 additions
differs); the dequantised, SwiGLU and bf16 outputs within that bound carried
through their arithmetic; the blocks within 1e-2 max-relative of the oracle.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import LINEAR_CONFIGS, MOE_CONFIGS, linear_inputs, moe_inputs
from synthetic.workloads import DIT_LINEARS, MoEConfig
from tests.code_budget import check_codes
from tests.lowbit_format import unpack_lowbit

pytestmark = pytest.mark.gpu

W = None


@pytest.fixture(scope="module", autouse=True)
def gpu_lib():
    global W
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import w8a8_rotated_int8_b200 as lib_mod
    lib_mod.load_library()
    lib_mod.convrot_device_check()
    W = lib_mod
    yield
    W.convrot_check_device_error()


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert W.convrot_check_device_error() == 0


def np32(t):
    return t.detach().float().cpu().numpy()


def _bf16_weights(rows, k, seed, special_rows=True):
    gen = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, k, generator=gen) * 0.02
    w[:, torch.randperm(k, generator=gen)[: max(1, k // 100)]] *= 10   # outlier columns
    if special_rows and rows >= 4:
        w[0] = 0.0                      # zero row: s_r = 0, every code 0
        w[1] *= 1e-33                   # tiny row: s_r an fp32 subnormal
        w[2, : k // 2] *= 1e-6          # groups far below the row maximum
    return w.to(torch.bfloat16)


def _unpacked(lw):
    q, sig = unpack_lowbit(lw.data.cpu().numpy(), lw.n_mats * lw.rows, lw.k, lw.bits)
    return q, sig, lw.scale.cpu().numpy()


# ------------------------------------------------------------- quantiser --
@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("rows,k,g", [(256, 512, 256), (384, 2048, 256), (128, 1536, 64),
                                      (256, 3840, 256), (128, 64, 16), (128, 256, 1),
                                      (128, 320, 64), (128, 16384, 256)])
def test_lowbit_weight_quantisation_bit_exact(bits, rows, k, g):
    w = _bf16_weights(rows, k, seed=rows + k + g + bits)
    lw = W.convrot_quantize_weights_lowbit(w.cuda(), g, bits)
    q, sig, s_r = _unpacked(lw)
    q_ref, sig_ref, s_ref = O.rotquant_lowbit(np32(w), g, bits)
    assert np.array_equal(s_r, s_ref)
    assert np.array_equal(sig, sig_ref)
    assert np.array_equal(q, q_ref)


def test_lowbit_weight_bytes_and_checks():
    assert W.lowbit_weight_bytes(256, 2048, 4) == 2 * 32 * 4608
    assert W.lowbit_weight_bytes(256, 2048, 6) == 2 * 32 * 6656
    assert W.lowbit_weight_bytes(100, 2048, 4) == -1
    w = _bf16_weights(128, 96, 1).cuda()
    with pytest.raises((ValueError, W.ConvrotError)):   # K % 64
        W.convrot_quantize_weights_lowbit(w, 16, 4)


# ------------------------------------------------------------------ GEMM --
def _codes(shape, seed, lo=-127, hi=128):
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi, shape, generator=gen, dtype=torch.int8)


def _gemm_case(g, m, n, k, bits, seed, group=256):
    x = _codes((g, m, k), seed)
    s_x = torch.rand(g, m, generator=torch.Generator().manual_seed(seed + 1)) * 0.05 + 1e-3
    w = _bf16_weights(g * n, k, seed + 2, special_rows=False)
    lw = W.convrot_quantize_weights_lowbit(w.cuda(), group if k % group == 0 else 64, bits,
                                           n_mats=g)
    q, sig, s_r = _unpacked(lw)
    return x, s_x, lw, q.reshape(g, n, k), sig.reshape(g, n, k // 16), s_r.reshape(g, n)


def _acc_ref_and_bound(x, q, sig):
    """Exact acc per group and the bound of an fp32 summation of its terms."""
    xs = x.numpy().astype(np.float64)
    wq = q.astype(np.float64) * np.repeat(O.e4m3_decode(sig), 16, axis=-1)
    acc = np.stack([O.lowbit_acc(x[i].numpy(), q[i], sig[i]) for i in range(x.shape[0])])
    mag = np.stack([np.abs(xs[i]) @ np.abs(wq[i]).T for i in range(x.shape[0])])
    k = x.shape[-1]
    return acc, k * 2.0 ** -23 * mag + 1e-30


GEMM_CASES = [  # g, m, n, k, tile_tokens (0 = the library's choice)
    (1, 64, 256, 256, 0), (3, 100, 512, 384, 0), (2, 200, 256, 2048, 0), (2, 200, 256, 512, 64),
    (1, 33, 768, 192, 16), (2, 130, 256, 320, 128), (1, 1, 256, 64, 0), (2, 256, 512, 1536, 0),
    (1, 48, 256, 640, 48),
    # more than 128 tokens per group with the library's choice: CTA pairs of
    # 2 x 128 tokens (one over, ragged second CTA, several pair blocks)
    (3, 129, 256, 128, 0), (2, 300, 768, 640, 0), (1, 520, 512, 256, 0),
]


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("g,m,n,k,nt", GEMM_CASES)
def test_lowbit_gemm_accumulator(bits, g, m, n, k, nt):
    x, s_x, lw, q, sig, s_r = _gemm_case(g, m, n, k, bits, seed=g * 1000 + m + n + k)
    acc = W.convrot_lowbit_gemm(x.cuda(), None, lw, W.CONVROT_LOWBIT_F32, nt)
    torch.cuda.synchronize()
    ref, bound = _acc_ref_and_bound(x, q, sig)
    err = np.abs(acc.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= bound), float((err / bound).max())


def test_lowbit_gemm_extremes():
    """Codes +-127 against weights whose every group has sigma = 448 and codes
    +-qmax: the largest products the format allows, K = 2048."""
    for bits in (4, 6):
        g, m, n, k = 1, 64, 256, 2048
        gen = torch.Generator().manual_seed(5)
        sign = torch.randint(0, 2, (n, k), generator=gen) * 2 - 1
        w = sign.float().to(torch.bfloat16)            # g = 1: every group's max is the row's
        lw = W.convrot_quantize_weights_lowbit(w.cuda(), 1, bits)
        q, sig, _ = _unpacked(lw)
        assert np.all(sig == 0x7E) and np.all(np.abs(q) == 2 ** (bits - 1) - 1)
        x = (torch.randint(0, 2, (g, m, k), generator=gen) * 254 - 127).to(torch.int8)
        acc = W.convrot_lowbit_gemm(x.cuda(), None, lw, W.CONVROT_LOWBIT_F32)
        ref, bound = _acc_ref_and_bound(x, q[None], sig[None])
        assert np.all(np.abs(acc.cpu().numpy() - ref) <= bound)


def _bf16_ulp(v):
    v = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(v)) - 7)


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("g,m,n,k,nt", [(2, 200, 512, 1024, 0), (1, 40, 256, 256, 0),
                                        (3, 77, 256, 384, 32), (1, 390, 768, 512, 0)])
def test_lowbit_gemm_bf16(bits, g, m, n, k, nt):
    x, s_x, lw, q, sig, s_r = _gemm_case(g, m, n, k, bits, seed=7 * m + n)
    y = W.convrot_lowbit_gemm(x.cuda(), s_x.cuda(), lw, W.CONVROT_LOWBIT_BF16, nt)
    ref, bound = _acc_ref_and_bound(x, q, sig)
    sx = s_x.numpy()
    for i in range(g):
        y32 = O.lowbit_dequant(ref[i], s_r[i], sx[i]).astype(np.float64)
        scale = np.abs(sx[i][:, None].astype(np.float64) * s_r[i][None, :])
        tol = bound[i] * scale * 1.001 + 2.0 ** -22 * np.abs(y32) + 0.5 * _bf16_ulp(y32) * 1.001
        got = np32(y[i]).astype(np.float64)
        assert np.all(np.abs(got - y32) <= tol)
        # nearly every output is the oracle's bf16 value itself
        same = np.mean(got == O.bf16_round(y32.astype(np.float32)))
        assert same > 0.97, same


def _check_swiglu(h_gpu, x_q, s_x, q, sig, s_r):
    """h from the GPU against the oracle's SwiGLU of the same codes: the fp32
    summation bound of both accumulators carried through silu(g) * u (|silu'|
    <= 1.1), plus a few fp32 ulp for CUDA expf and the division."""
    f = q.shape[0] // 2
    h_ref = O.lowbit_swiglu_from_codes(x_q, s_x, q, sig, s_r)
    ref, bound = _acc_ref_and_bound(torch.from_numpy(np.ascontiguousarray(x_q))[None], q[None],
                                    sig[None])
    y = O.lowbit_dequant(ref[0], s_r, s_x).astype(np.float64)
    dy = bound[0] * np.abs(s_x[:, None] * s_r[None, :]) * 1.001 + 2.0 ** -22 * np.abs(y)
    yg, yu = y[:, :f], y[:, f:]
    silu = yg / (1 + np.exp(-yg))
    tol = (1.1 * dy[:, :f] * np.abs(yu) + np.abs(silu) * dy[:, f:]
           + 8 * 2.0 ** -23 * np.abs(h_ref) + 1e-30)
    assert np.all(np.abs(np.asarray(h_gpu, np.float64) - h_ref) <= tol)


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("g,m,f,k,nt", [(2, 160, 256, 768, 0), (1, 64, 1536, 2048, 0),
                                        (3, 40, 128, 512, 16), (2, 280, 384, 256, 0)])
def test_lowbit_gemm_swiglu(bits, g, m, f, k, nt):
    x, s_x, lw, q, sig, s_r = _gemm_case(g, m, 2 * f, k, bits, seed=3 * m + f)
    h = W.convrot_lowbit_gemm(x.cuda(), s_x.cuda(), lw, W.CONVROT_LOWBIT_SWIGLU, nt)
    for i in range(g):
        _check_swiglu(np32(h[i]), x[i].numpy(), s_x[i].numpy(), q[i], sig[i], s_r[i])


def test_lowbit_gemm_rejects_bad_shapes():
    x = torch.zeros(1, 64, 256, dtype=torch.int8, device="cuda")
    w = W.convrot_quantize_weights_lowbit(_bf16_weights(128, 256, 3).cuda(), 256, 4)
    with pytest.raises(W.ConvrotError):     # N = 128 is not a multiple of 256
        W.convrot_lowbit_gemm(x, None, w, W.CONVROT_LOWBIT_F32)


# --------------------------------------------------------------- linears --
def _linear_case(name):
    if name in LINEAR_CONFIGS:
        cfg = LINEAR_CONFIGS[name]
        x, w = linear_inputs(cfg)
        return x, w, cfg.group
    spec = DIT_LINEARS[name]
    x, w = linear_inputs(spec)
    return x, w, spec.group


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("name", ["linear_64x256x256", "gateup_4096x3072x2048",
                                  "down_4096x2048x1536", "dit_adaln", "dit_out", "dit_ffn_down"])
def test_lowbit_linear(bits, name):
    """End to end through lowbit_convrot_linear: weights bit-exact; all
    activation codes within the budget of the definition; sampled output rows
    against the oracle given the same codes (fp32 summation bound + bf16
    rounding) and within 1e-2 of the oracle's whole linear."""
    x, w, g = _linear_case(name)
    lw = W.convrot_quantize_weights_lowbit(w.cuda(), g, bits)
    y = W.lowbit_convrot_linear(x.cuda(), lw, g)
    xq, sx = W.convrot_rotquant(x.cuda(), g)
    xq_np, sx_np = xq.cpu().numpy(), sx.cpu().numpy()
    check_codes(xq_np, sx_np, np32(x), g)
    q, sig, s_r = _unpacked(lw)
    q_ref, sig_ref, s_ref = O.rotquant_lowbit(np32(w), g, bits)
    assert np.array_equal(q, q_ref) and np.array_equal(sig, sig_ref)
    assert np.array_equal(s_r, s_ref)
    m = x.shape[0]
    rows = np.arange(m) if m <= 256 else np.unique(np.random.default_rng(0).integers(0, m, 64))
    ref, bound = _acc_ref_and_bound(torch.from_numpy(xq_np[rows])[None], q[None], sig[None])
    y32 = O.lowbit_dequant(ref[0], s_r, sx_np[rows]).astype(np.float64)
    tol = (bound[0] * np.abs(sx_np[rows][:, None] * s_r[None, :]) * 1.001
           + 2.0 ** -22 * np.abs(y32) + 0.5 * _bf16_ulp(y32) * 1.001)
    got = np32(y)[rows].astype(np.float64)
    assert np.all(np.abs(got - y32) <= tol)
    y_full = O.lowbit_linear(np32(x)[rows], q, sig, s_r, g)
    assert np.max(np.abs(got - y_full)) <= 1e-2 * np.max(np.abs(y_full))


# ------------------------------------------------------------- MoE block --
LB_MOE = {
    "moe_lb_small": MoEConfig("moe_lb_small", 640, 768, 6, 384, 160, 31),
    "moe_lb_c40": MoEConfig("moe_lb_c40", 300, 512, 5, 256, 40, 32),
    "moe_lb_gd16": MoEConfig("moe_lb_gd16", 200, 256, 3, 128, 96, 33, g_gu=64, g_d=16),
}


def _run_lowbit_moe(inp, cfg, bits):
    gu, dn = W.quantize_moe_weights_lowbit(inp["wgu"].cuda(), inp["wd"].cuda(), bits,
                                           cfg.g_gu, cfg.g_d)
    ws = torch.empty(W.moe_workspace_size(cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c),
                     dtype=torch.uint8, device="cuda")
    y = W.moe_expert_choice_forward_lowbit(inp["x"].cuda(), inp["logits"].cuda(), gu, dn, cfg.c,
                                           cfg.g_gu, cfg.g_d, workspace=ws)
    torch.cuda.synchronize()
    views = W.moe_stage_views(ws, cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c)
    return y, views, gu, dn


def _lowbit_moe_weights(gu, dn, cfg):
    e = cfg.n_exp
    qg, sg, rg = _unpacked(gu)
    qd, sd, rd = _unpacked(dn)
    return ((qg.reshape(e, 2 * cfg.f, cfg.d), sg.reshape(e, 2 * cfg.f, cfg.d // 16),
             rg.reshape(e, 2 * cfg.f)),
            (qd.reshape(e, cfg.d, cfg.f), sd.reshape(e, cfg.d, cfg.f // 16), rd.reshape(e, cfg.d)))


def _check_lowbit_stages(v, cfg, idx, w, gu_ref, dn_ref, experts):
    """Each stage given the GPU's own inputs to it: gather exact; h within the
    SwiGLU bound of the oracle's from the gathered codes; h codes within the
    budget; z within the summation bound of the oracle's from the h codes."""
    x_q, s_x = v["x_q"].cpu().numpy(), v["s_x"].cpu().numpy()
    assert np.array_equal(v["idx"].cpu().numpy(), idx)
    assert np.array_equal(v["w"].cpu().numpy(), w)
    assert np.array_equal(v["x_g"].cpu().numpy(), x_q[idx])
    flips = codes = 0
    for e in experts:
        rows = idx[e]
        h = v["h"][e].cpu().numpy()
        _check_swiglu(h, x_q[rows], s_x[rows], gu_ref[0][e], gu_ref[1][e], gu_ref[2][e])
        h_q, s_h = v["h_q"][e].cpu().numpy(), v["s_h"][e].cpu().numpy()
        n, c, _, _ = check_codes(h_q, s_h, h, cfg.g_d)
        flips, codes = flips + n, codes + c
        ref, bound = _acc_ref_and_bound(torch.from_numpy(h_q)[None], dn_ref[0][e][None],
                                        dn_ref[1][e][None])
        z32 = O.lowbit_dequant(ref[0], dn_ref[2][e], s_h).astype(np.float64)
        tol = (bound[0] * np.abs(s_h[:, None] * dn_ref[2][e][None, :]) * 1.001
               + 2.0 ** -22 * np.abs(z32) + 0.5 * _bf16_ulp(z32) * 1.001)
        assert np.all(np.abs(np32(v["z"][e]).astype(np.float64) - z32) <= tol)
    return flips, codes


@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("name", sorted(LB_MOE))
def test_lowbit_moe_block_small(bits, name):
    cfg = LB_MOE[name]
    inp = moe_inputs(cfg)
    y, v, gu, dn = _run_lowbit_moe(inp, cfg, bits)
    gu_ref, dn_ref = _lowbit_moe_weights(gu, dn, cfg)
    # offline weights bit-exact against the oracle's quantiser
    for e in range(cfg.n_exp):
        q, s, r = O.rotquant_lowbit(np32(inp["wgu"][e]), cfg.g_gu, bits)
        assert np.array_equal(q, gu_ref[0][e]) and np.array_equal(s, gu_ref[1][e])
        assert np.array_equal(r, gu_ref[2][e])
        q, s, r = O.rotquant_lowbit(np32(inp["wd"][e]), cfg.g_d, bits)
        assert np.array_equal(q, dn_ref[0][e]) and np.array_equal(s, dn_ref[1][e])
        assert np.array_equal(r, dn_ref[2][e])
    x_np, logits_np = np32(inp["x"]), np32(inp["logits"])
    y_ref, it = O.moe_block_lowbit(x_np, logits_np, gu_ref, dn_ref, cfg.c, cfg.g_gu, cfg.g_d,
                                   keep=True)
    check_codes(v["x_q"].cpu().numpy(), v["s_x"].cpu().numpy(), x_np, cfg.g_gu)
    _check_lowbit_stages(v, cfg, it["idx"], it["w"], gu_ref, dn_ref, range(cfg.n_exp))
    z = {e: np32(v["z"][e]) for e in range(cfg.n_exp)}
    y_np = np32(y)
    assert np.array_equal(y_np, O.combine(cfg.t, it["idx"], it["w"], z))
    assert np.max(np.abs(y_np - y_ref)) <= 1e-2 * np.max(np.abs(y_ref))


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 6])
@pytest.mark.parametrize("name", ["moe_T2048", "moe_T8192"])
def test_lowbit_moe_block_full_size(bits, name):
    """The T=2048 and T=8192 blocks in the bench's launch configuration (64
    and 256 tokens per expert: single CTAs and CTA pairs): routing exact,
    every stage of a spread of experts against the oracle given the GPU's
    inputs to it, every output row given z, and sampled rows within 1e-2 of
    the oracle's whole block."""
    cfg = MOE_CONFIGS[name]
    inp = moe_inputs(cfg)
    y, v, gu, dn = _run_lowbit_moe(inp, cfg, bits)
    gu_ref, dn_ref = _lowbit_moe_weights(gu, dn, cfg)
    experts = [0, 17, 42, 63]
    for e in experts:
        q, s, r = O.rotquant_lowbit(np32(inp["wgu"][e]), cfg.g_gu, bits)
        assert np.array_equal(q, gu_ref[0][e]) and np.array_equal(s, gu_ref[1][e])
        q, s, r = O.rotquant_lowbit(np32(inp["wd"][e]), cfg.g_d, bits)
        assert np.array_equal(q, dn_ref[0][e]) and np.array_equal(r, dn_ref[2][e])
    x_np, logits_np = np32(inp["x"]), np32(inp["logits"])
    idx, w = O.expert_choice_topc(O.router_softmax(logits_np), cfg.c)
    _check_lowbit_stages(v, cfg, idx, w, gu_ref, dn_ref, experts)
    z = {e: np32(v["z"][e]) for e in range(cfg.n_exp)}
    y_np = np32(y)
    assert np.array_equal(y_np, O.combine(cfg.t, idx, w, z))
    sample = np.unique(np.concatenate([np.arange(6), np.random.default_rng(1).choice(
        cfg.t, 10, replace=False)]))
    y_ref = O.moe_block_lowbit(x_np, logits_np, gu_ref, dn_ref, cfg.c, cfg.g_gu, cfg.g_d,
                               out_tokens=sample)
    assert np.max(np.abs(y_np[sample] - y_ref[sample])) <= 1e-2 * np.max(np.abs(y_ref[sample]))
