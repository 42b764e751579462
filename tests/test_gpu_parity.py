"""GPU parity: every stage of the CUDA path through the C ABI against the oracle.

Bar: bit-exact weight codes and scales (fp64 offline quantiser), int32
accumulators, top-C index sets, dequantised outputs and the router-weighted
combine, each given the same quantised inputs; the run-time activation and h
codes (fp32 rotation) within the budget of tests/code_budget.py (at most 1e-4
of the codes one off, only next to a half-integer, none further); the SwiGLU
output and the atomic scatter epilogue within the bounds their arithmetic
allows (CUDA expf vs a correctly rounded exp; atomic accumulation order); the
block output within the 1e-2 max-relative budget.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import LINEAR_CONFIGS, MOE_CONFIGS, linear_inputs, moe_inputs
from tests.code_budget import check_codes
from tests.golden import read_fixture

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


def bf16_activations(rows, k, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, k, generator=g)
    if outliers:
        ch = torch.randperm(k, generator=g)[: max(1, round(0.01 * k))]
        x[:, ch] *= 20
    return x.to(torch.bfloat16)


# ----------------------------------------------------------- rotate+quant --
@pytest.mark.parametrize("rows,k,g", [
    (64, 256, 256), (300, 768, 256), (257, 2048, 256), (5, 8192, 256), (33, 320, 64),
    (100, 1536, 64), (77, 512, 16), (50, 256, 4), (40, 64, 1), (3, 16, 16), (1, 4096, 64),
    (20000, 2048, 256),  # many more row groups than resident CTAs (persistent loop)
])
def test_rotquant_bf16_within_budget(rows, k, g):
    x = bf16_activations(rows, k, seed=rows * 7 + k)
    q, s = W.convrot_rotquant(x.cuda(), g)
    check_codes(q.cpu().numpy(), s.cpu().numpy(), np32(x), g)


@pytest.mark.parametrize("rows,k,g", [(160, 320, 64), (513, 1536, 64), (64, 2048, 256),
                                      (9001, 1536, 64), (3, 192, 64), (11, 8192 - 64, 64)])
def test_rotquant_f32_within_budget(rows, k, g):
    """fp32 rows (the SwiGLU output); K = 320, 1536, 192, 8128 have group
    counts that are not powers of two (one thread per group); the first row
    is zero and the second tiny (absmax about 1e-38, below the reciprocal's
    range: its codes come from the subnormal-capable scale)."""
    gen = torch.Generator().manual_seed(k)
    a = torch.randn(rows, k, generator=gen)
    b = torch.randn(rows, k, generator=gen)
    h = (torch.nn.functional.silu(a) * b).float()  # SwiGLU-shaped fp32 rows
    h[0] = 0.0
    if rows > 1:
        h[1] = h[1] * 1e-38
    q, s = W.convrot_rotquant(h.cuda(), g)
    check_codes(q.cpu().numpy(), s.cpu().numpy(), h.numpy(), g)
    assert float(s[0]) == 0.0 and int(q[0].abs().sum()) == 0


def test_rotquant_subnormal_scale_worked_example():
    """The oracle's hand-worked tiny row (g = 1): a = 2^-140 gives the
    subnormal s = 2^-147, and the codes 2^-140 / s = 128 and -128 clamp to
    +-127 while -2^-141 / s = -64; a = 2^-145 gives s = 0 and zero codes."""
    v = torch.zeros(3, 16)
    v[1, 2], v[1, 5], v[1, 6] = 2.0 ** -140, -(2.0 ** -141), -(2.0 ** -140)
    v[2, 0] = 2.0 ** -145
    q, s = W.convrot_rotquant(v.cuda(), 1)
    q, s = q.cpu(), s.cpu()
    assert float(s[1]) == 2.0 ** -147
    assert q[1, :8].tolist() == [0, 0, 127, 0, 0, -64, -127, 0]
    assert float(s[0]) == 0.0 and float(s[2]) == 0.0
    assert int(q[0].abs().sum()) == 0 and int(q[2].abs().sum()) == 0
    q_ref, s_ref = O.rotquant(v.numpy(), 1)
    assert np.array_equal(q.numpy(), q_ref) and np.array_equal(s.numpy(), s_ref)


def test_rotquant_worked_examples_and_degenerate_rows():
    ties = read_fixture("quant_ties.txt")
    rot = read_fixture("rotation_g4.txt")
    x = torch.zeros(4, 16)
    x[0, :8] = torch.tensor(ties["input"][0])
    x[1, :8] = torch.tensor(rot["input"][0])
    x[3, :] = 0.75  # constant row
    xb = x.to(torch.bfloat16)
    q1, s1 = W.convrot_rotquant(xb.cuda(), 1)
    assert q1[0, :8].tolist() == ties["codes"][0] and s1[0].item() == 1.0
    assert q1[2].abs().sum().item() == 0 and s1[2].item() == 0.0  # zero row
    q4, s4 = W.convrot_rotquant(xb.cuda(), 4)
    assert q4[1, :8].tolist() == rot["codes"][0]
    assert s4[1].item() == np.float32(13.0 / 127.0)
    assert q4[2].abs().sum().item() == 0


@pytest.mark.parametrize("rows,k,g", [(300, 768, 256), (64, 8192, 256), (1000, 1536, 64),
                                      (77, 512, 16), (50, 256, 4), (40, 64, 1), (3, 16, 16)])
def test_weight_quantisation_bit_exact(rows, k, g):
    """The offline quantiser (fp64 rotation and quotients) equals the
    definition bit for bit: codes and scales, on outlier-laden rows too."""
    w = bf16_activations(rows, k, seed=rows + 3 * k)
    w = (w.float() * 0.02).to(torch.bfloat16)
    q, s = W.convrot_quantize_weights(w.cuda(), g)
    q_ref, s_ref = O.rotquant(np32(w), g)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_weight_quantisation_3d_stack():
    cfg = MOE_CONFIGS["moe_small"]
    inp = moe_inputs(cfg)
    q, s = W.convrot_quantize_weights(inp["wd"].cuda(), cfg.g_d)
    for e in range(cfg.n_exp):
        q_ref, s_ref = O.rotquant(np32(inp["wd"][e]), cfg.g_d)
        assert np.array_equal(q[e].cpu().numpy(), q_ref)
        assert np.array_equal(s[e].cpu().numpy(), s_ref)


# ----------------------------------------------------------------- routing --
def _ulp_diff(a, b):
    ai = a.view(np.int32).astype(np.int64)
    bi = b.view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


@pytest.mark.parametrize("t,e", [(8192, 64), (1000, 8), (33, 256), (1, 1), (500, 100),
                                 (77, 200)])
def test_router_softmax(t, e):
    gen = torch.Generator().manual_seed(t + e)
    logits = torch.randn(t, e, generator=gen).to(torch.bfloat16)
    s_t = W.convrot_router_softmax(logits.cuda()).cpu().numpy()
    ref = O.router_softmax(np32(logits)).T
    d = _ulp_diff(s_t, ref)
    assert d.max() <= 1
    assert (d != 0).mean() <= 1e-4


# T <= 1024, 2048, 4096, 8192, 16384 scores per expert use the register-resident
# kernel with 1, 2, 4, 8, 16 tokens per thread (vector loads when T % 4 == 0);
# larger T the general one
@pytest.mark.parametrize("t,e,c", [(8192, 64, 256), (2048, 64, 64), (1000, 8, 100),
                                   (300, 5, 300), (50, 3, 1), (1, 2, 1), (64, 4, 0),
                                   (16384, 2, 512), (8190, 3, 255), (5000, 4, 700),
                                   (20000, 3, 600), (4097, 2, 4097)])
def test_topc_exact_given_scores(t, e, c):
    gen = torch.Generator().manual_seed(t * 3 + c)
    s = torch.softmax(torch.randn(t, e, generator=gen), dim=1).numpy().astype(np.float32)
    if t in (1000, 5000, 20000):
        s = (np.floor(s * 16) / 16).astype(np.float32)  # heavy ties
    idx, w = W.convrot_topc(torch.from_numpy(np.ascontiguousarray(s.T)).cuda(), c)
    idx_ref, w_ref = O.expert_choice_topc(s, c)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.array_equal(w.cpu().numpy(), w_ref)


@pytest.mark.parametrize("t,c", [(700, 90), (8192, 256), (3001, 77), (17000, 300)])
def test_topc_slot_table_inverts_idx(t, c):
    gen = torch.Generator().manual_seed(5 + t)
    s = torch.softmax(torch.randn(t, 6, generator=gen), dim=1).numpy().astype(np.float32)
    idx, w, slot = W.convrot_topc(torch.from_numpy(np.ascontiguousarray(s.T)).cuda(), c,
                                  with_slot=True)
    idx, slot = idx.cpu().numpy(), slot.cpu().numpy()
    expect = np.full((6, t), -1, np.int32)
    for e in range(6):
        expect[e, idx[e]] = np.arange(c)
    assert np.array_equal(slot, expect)


def _degenerate_scores(kind, t, e, gen):
    if kind == "equal":  # every token ties: the first C tokens win
        return np.full((t, e), 0.25, np.float32)
    if kind == "signed_zero":  # -0 and +0 compare equal
        z = np.where(torch.rand(t, e, generator=gen).numpy() < 0.5, -0.0, 0.0).astype(np.float32)
        z[::7] = 1e-3
        return z
    if kind == "signed":  # negative scores, +-inf and subnormals order by value
        s = torch.randn(t, e, generator=gen).numpy().astype(np.float32)
        s[::5] = np.float32(1e-40) * np.sign(s[::5])
        s[3::11] = np.inf
        s[4::13] = -np.inf
        return s
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["equal", "signed_zero", "signed"])
@pytest.mark.parametrize("t", [1, 31, 1000, 4096, 16384])
def test_topc_degenerate_scores(kind, t):
    """Degenerate score columns: all equal, signed zeros, negatives, +-inf,
    subnormals; C in {0, 1, T // 3, T}. The picks equal the oracle's and the
    slot table inverts them."""
    e = 3
    gen = torch.Generator().manual_seed(t + len(kind))
    s = _degenerate_scores(kind, t, e, gen)
    s_dev = torch.from_numpy(np.ascontiguousarray(s.T)).cuda()
    for c in sorted({0, 1, t // 3, t}):
        idx, w, slot = W.convrot_topc(s_dev, c, with_slot=True)
        idx_ref, w_ref = O.expert_choice_topc(s, c)
        idx, w, slot = idx.cpu().numpy(), w.cpu().numpy(), slot.cpu().numpy()
        assert np.array_equal(idx, idx_ref), (kind, t, c)
        assert np.array_equal(w, w_ref), (kind, t, c)  # by value: a -0 pick comes back as +0
        expect = np.full((e, t), -1, np.int32)
        for x in range(e):
            expect[x, idx[x]] = np.arange(c)
        assert np.array_equal(slot, expect), (kind, t, c)


def test_gather_rows():
    src = torch.randint(-127, 128, (100, 64), dtype=torch.int8)
    s_src = torch.rand(100)
    idx = torch.tensor([5, 0, 99, 5, 42], dtype=torch.int32)
    dst, s_dst = W.convrot_gather_rows(src.cuda(), s_src.cuda(), idx.cuda())
    assert torch.equal(dst.cpu(), src[idx.long()])
    assert torch.equal(s_dst.cpu(), s_src[idx.long()])


# -------------------------------------------------------------------- GEMM --
GEMM_SHAPES = [(1, 64, 256, 256), (3, 160, 320, 768), (2, 40, 48, 2048), (1, 128, 256, 128),
               (1, 300, 272, 1536), (4, 256, 3072, 2048), (1, 1, 16, 16), (2, 129, 512, 64),
               # groups of <= 128 rows with >= 148 single-CTA tiles run on CTA pairs
               (40, 64, 1024, 512), (150, 100, 256, 128)]


def _codes(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int8)


def _tiled_codes(b):
    """Place row-major codes [G, N, K] in the tiled weight format (test-side,
    plain tensor reshapes) and wrap them like convrot_quantize_weights_tiled."""
    g, n, k = b.shape
    rb, kb = -(-n // 128), -(-k // 128)
    pad = torch.zeros((g, rb * 128, kb * 128), dtype=torch.int8)
    pad[:, :n, :k] = b
    data = pad.view(g, rb, 128, kb, 128).permute(0, 1, 3, 2, 4).contiguous().view(-1)
    return W.TiledWeights(data.cuda(), None, g, n, k)


@pytest.mark.parametrize("layout", ["rows", "tiles"])
@pytest.mark.parametrize("g,m,n,k", GEMM_SHAPES)
def test_gemm_int32_bit_exact(g, m, n, k, layout):
    a = _codes((g, m, k), 1 + m)
    b = _codes((g, n, k), 2 + n)
    bb = b.cuda() if layout == "rows" else _tiled_codes(b)
    d = W.convrot_i8_gemm_i32(a.cuda(), bb).cpu().numpy()
    for gi in range(g):
        assert np.array_equal(d[gi], O.int_gemm(a[gi].numpy(), b[gi].numpy()))


def test_tiled_weight_quantisation_matches_row_major():
    w = bf16_activations(3 * 200, 320, seed=5)
    rows_q, rows_s = W.convrot_quantize_weights(w.cuda(), 64)
    tw = W.convrot_quantize_weights_tiled(w.cuda(), 64, n_mats=3)
    assert torch.equal(W.untile(tw), rows_q)
    assert torch.equal(tw.scale, rows_s)
    # padding rows (200..255 of each matrix) and columns (320..383) are zero
    full = tw.data.view(3, 2, 3, 128, 128)
    assert int(full[:, 1, :, 72:, :].abs().sum()) == 0
    assert int(full[:, :, 2, :, 64:].abs().sum()) == 0


def test_gemm_int32_extremes():
    k = 2048
    a = torch.full((1, 128, k), 127, dtype=torch.int8)
    b = torch.full((1, 256, k), -127, dtype=torch.int8)
    b[0, 1] = 127
    d = W.convrot_i8_gemm_i32(a.cuda(), b.cuda()).cpu()
    assert int(d[0, 0, 0]) == -k * 127 * 127 and int(d[0, 5, 1]) == k * 127 * 127


@pytest.mark.parametrize("g,m,n,k", [(1, 64, 256, 256), (2, 200, 320, 512), (1, 513, 528, 1536),
                                     (40, 64, 1024, 512)])
def test_gemm_bf16_dequant_bit_exact(g, m, n, k):
    a = _codes((g, m, k), 3)
    b = _codes((g, n, k), 4)
    s_a = torch.rand(g, m) * 0.05 + 1e-3
    s_b = torch.rand(g, n) * 1e-3 + 1e-5
    y = W.convrot_i8_gemm_bf16(a.cuda(), s_a.cuda(), b.cuda(), s_b.cuda()).cpu()
    for gi in range(g):
        ref = O.bf16_round(O.dequant(O.int_gemm(a[gi].numpy(), b[gi].numpy()),
                                     s_b[gi].numpy(), s_a[gi].numpy()))
        assert np.array_equal(np32(y[gi]), ref)


def _fp32_ulps(x, ref):
    return np.abs(x.astype(np.float64) - ref) / np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)


@pytest.mark.parametrize("layout", ["rows", "tiles"])
@pytest.mark.parametrize("g,m,f,k", [(2, 160, 320, 768), (1, 64, 1536, 2048), (3, 40, 192, 512),
                                     (40, 64, 512, 256)])
def test_gemm_swiglu(g, m, f, k, layout):
    a = _codes((g, m, k), 5)
    b = _codes((g, 2 * f, k), 6)
    s_a = torch.rand(g, m) * 0.05 + 1e-3
    s_b = torch.rand(g, 2 * f) * 1e-4 + 1e-6
    bb = b.cuda() if layout == "rows" else _tiled_codes(b.view(2 * g, f, k))
    h = W.convrot_i8_gemm_swiglu(a.cuda(), s_a.cuda(), bb, s_b.cuda()).cpu().numpy()
    for gi in range(g):
        y = O.dequant(O.int_gemm(a[gi].numpy(), b[gi].numpy()), s_b[gi].numpy(), s_a[gi].numpy())
        ref = (O.silu_f32(y[:, :f]) * y[:, f:]).astype(np.float32)
        ulps = _fp32_ulps(h[gi], ref)
        # CUDA expf is within 2 ulp of exp: silu(g)*u within a few ulp
        assert ulps.max() <= 4
        assert (ulps == 0).mean() > 0.8  # expf differs from exp in ~1 of 10 elements


# The requantising SwiGLU epilogue: h rotated and quantised per row inside the
# GEMM. Shapes cover the single-CTA and the CTA-pair kernels, a last tile with
# one half of its h columns (F % 128 = 64) or a part of one (F % 64 = 16),
# a pair m-block whose second slab holds no row, more tiles than resident
# CTAs (row blocks spread over two tiles of one CTA's loop) and every group.
@pytest.mark.parametrize("layout", ["rows", "tiles"])
@pytest.mark.parametrize("g,m,f,k,g_h", [
    (2, 160, 320, 768, 64), (1, 64, 1536, 2048, 64), (3, 40, 192, 512, 16),
    (2, 300, 256, 256, 4), (5, 100, 208, 256, 16), (40, 64, 512, 256, 64),
    (3, 130, 64, 128, 1), (24, 256, 1536, 256, 64),
])
def test_gemm_swiglu_rq_matches_two_step(g, m, f, k, g_h, layout):
    """Codes and scales equal the SwiGLU GEMM followed by the rotation kernel
    bit for bit (the same fp32 arithmetic), and the definition's codes of
    that same h within the budget."""
    a = _codes((g, m, k), 7 + m)
    b = _codes((g, 2 * f, k), 8 + f)
    s_a = (torch.rand(g, m) * 0.05 + 1e-3).cuda()
    s_b = (torch.rand(g, 2 * f) * 1e-4 + 1e-6).cuda()
    bb = b.cuda() if layout == "rows" else _tiled_codes(b.view(2 * g, f, k))
    s_a[0, 3] = 0.0  # an all-zero row of h: scale 0, codes 0
    h = W.convrot_i8_gemm_swiglu(a.cuda(), s_a, bb, s_b)
    q2, s2 = W.convrot_rotquant(h.view(-1, f), g_h)
    q1, s1 = W.convrot_i8_gemm_swiglu_rq(a.cuda(), s_a, bb, s_b, g_h)
    assert torch.equal(q1.view(-1, f), q2)
    assert torch.equal(s1.view(-1), s2)
    assert float(s1[0, 3]) == 0.0 and int(q1[0, 3].abs().sum()) == 0
    # and the definition's codes of that same h within the budget
    check_codes(q1.view(-1, f).cpu().numpy(), s1.view(-1).cpu().numpy(),
                h.view(-1, f).cpu().numpy(), g_h)


def test_gemm_swiglu_rq_repeated_calls_reuse_nothing():
    """Back-to-back calls on one stream (each clears its own scratch) give the
    same codes; a different input right after gives its own."""
    g, m, f, k = 6, 200, 384, 512
    a = _codes((g, m, k), 21).cuda()
    b = _codes((g, 2 * f, k), 22)
    bb = _tiled_codes(b.view(2 * g, f, k))
    s_a = (torch.rand(g, m) * 0.05 + 1e-3).cuda()
    s_b = (torch.rand(g, 2 * f) * 1e-4 + 1e-6).cuda()
    first = W.convrot_i8_gemm_swiglu_rq(a, s_a, bb, s_b, 64)
    for _ in range(3):
        again = W.convrot_i8_gemm_swiglu_rq(a, s_a, bb, s_b, 64)
        assert torch.equal(again[0], first[0]) and torch.equal(again[1], first[1])
    other = W.convrot_i8_gemm_swiglu_rq(a, s_a * 2, bb, s_b, 64)
    h = W.convrot_i8_gemm_swiglu(a, s_a * 2, bb, s_b)
    q2, s2 = W.convrot_rotquant(h.view(-1, f), 64)
    assert torch.equal(other[0].view(-1, f), q2) and torch.equal(other[1].view(-1), s2)


@pytest.mark.parametrize("layout", ["rows", "tiles"])
def test_gemm_scatter(layout):
    g, m, n, k, t = 4, 100, 320, 512, 150
    a = _codes((g, m, k), 7)
    b = _codes((g, n, k), 8)
    s_a = torch.rand(g, m) * 0.05 + 1e-3
    s_b = torch.rand(g, n) * 1e-4 + 1e-6
    gen = torch.Generator().manual_seed(9)
    idx = torch.stack([torch.sort(torch.randperm(t, generator=gen)[:m]).values for _ in range(g)])
    idx = idx.to(torch.int32)
    w = torch.rand(g, m)
    out = torch.zeros(t, n)
    ref = np.zeros((t, n), np.float32)
    for gi in range(g):
        z = O.dequant(O.int_gemm(a[gi].numpy(), b[gi].numpy()), s_b[gi].numpy(), s_a[gi].numpy())
        ref[idx[gi].numpy()] += w[gi].numpy()[:, None] * z
    bb = b.cuda() if layout == "rows" else _tiled_codes(b)
    out_gpu = W.convrot_i8_gemm_scatter(a.cuda(), s_a.cuda(), bb, s_b.cuda(), idx.cuda(),
                                        w.cuda(), out.cuda()).cpu().numpy()
    # fp32 sums of <= 4 terms in another order: within 4 ulps of the largest term
    assert np.max(np.abs(out_gpu - ref)) <= 4 * np.spacing(np.float32(np.abs(ref).max()))


@pytest.mark.parametrize("layout", ["rows", "tiles"])
@pytest.mark.parametrize("g,m", [(3, 100), (2, 300)])
def test_gemm_bf16_grouped_rows_bit_exact(g, m, layout):
    """The experts' down projection: grouped bf16 output rows in (group, row)
    order, through the 1-CTA (M <= 128) and the CTA-pair (M > 128) kernels."""
    n, k = 320, 512
    a = _codes((g, m, k), 10)
    b = _codes((g, n, k), 11)
    s_a = torch.rand(g, m) * 0.05 + 1e-3
    s_b = torch.rand(g, n) * 1e-4 + 1e-6
    bb = b.cuda() if layout == "rows" else _tiled_codes(b)
    z = W.convrot_i8_gemm_bf16(a.cuda(), s_a.cuda(), bb, s_b.cuda()).cpu()
    for gi in range(g):
        ref = O.bf16_round(O.dequant(O.int_gemm(a[gi].numpy(), b[gi].numpy()),
                                     s_b[gi].numpy(), s_a[gi].numpy()))
        assert np.array_equal(np32(z[gi]), ref)


@pytest.mark.parametrize("e_n,t,c,d", [(5, 300, 40, 256), (7, 64, 64, 2056), (3, 50, 0, 64),
                                       (70, 1000, 30, 128), (64, 5000, 160, 2048),
                                       (9, 40, 40, 8192), (200, 300, 250, 64)])
def test_combine_sums_in_expert_order(e_n, t, c, d):
    """y[t] = bf16(sum_e fp32(s_t[e, t] * z[e, slot])) in ascending expert order.
    d = 2056 leaves a ragged tail of 16-byte column vectors; d = 8192 gives
    every thread four column vectors; E = 200 with C = 250 of T = 300 gives
    tokens far more expert rows than one batch of loads covers."""
    gen = torch.Generator().manual_seed(3 + d)
    z = (torch.randn(e_n * c, d, generator=gen) * 10.0 ** torch.randint(-3, 3, (e_n * c, 1),
                                                                       generator=gen))
    z = z.to(torch.bfloat16)
    s_t = torch.rand(e_n, t, generator=gen)
    slot = torch.full((e_n, t), -1, dtype=torch.int32)
    for e in range(e_n):
        toks = torch.randperm(t, generator=gen)[:c].sort().values
        slot[e, toks] = torch.arange(c, dtype=torch.int32)
    y = W.convrot_combine_rows(z.cuda(), s_t.cuda(), slot.cuda(), c).cpu()
    # the same choices in the oracle's terms: each expert's tokens (ascending,
    # the slot order) and their router weights, and its rows of z
    idx = np.zeros((e_n, c), np.int32)
    zf, sf, sl = np32(z), s_t.numpy(), slot.numpy()
    for e in range(e_n):
        toks = np.nonzero(sl[e] >= 0)[0]
        idx[e, sl[e, toks]] = toks
    w = np.take_along_axis(sf, idx, axis=1).astype(np.float32)
    zd = {e: zf[e * c:(e + 1) * c] for e in range(e_n)}
    assert np.array_equal(np32(y), O.combine(t, idx, w, zd))


# ------------------------------------------------------------------ linear --
def _linear_with_codes(x, w_q, s_w, g):
    """The linear through its C-ABI entry, plus the activation codes and
    scales it left in its workspace."""
    m, k = x.shape
    ws = torch.empty(max(W.convrot_linear_workspace_size(m, k), 16), dtype=torch.uint8,
                     device="cuda")
    y = W.w8a8_convrot_linear(x, w_q, s_w, g, workspace=ws)
    torch.cuda.synchronize()
    x_q = ws[:m * k].view(torch.int8).view(m, k)
    off = (m * k + 255) // 256 * 256
    s_x = ws[off:off + 4 * m].view(torch.float32)
    return y, x_q, s_x


@pytest.mark.parametrize("name", ["linear_64x256x256", "gateup_4096x3072x2048",
                                  "down_4096x2048x1536"])
def test_w8a8_linear_parity(name):
    """Weights bit-exact; the output bit-exact given the GPU's activation codes;
    those codes within the budget; the output within 1e-2 of the oracle's."""
    cfg = LINEAR_CONFIGS[name]
    x, w = linear_inputs(cfg)
    w_q, s_w = W.convrot_quantize_weights(w.cuda(), cfg.group)
    y, x_q, s_x = _linear_with_codes(x.cuda(), w_q, s_w, cfg.group)
    w_q_ref, s_w_ref = O.rotquant(np32(w), cfg.group)
    assert np.array_equal(w_q.cpu().numpy(), w_q_ref) and np.array_equal(s_w.cpu().numpy(), s_w_ref)
    x_q, s_x = x_q.cpu().numpy(), s_x.cpu().numpy()
    assert np.array_equal(np32(y), O.w8a8_linear_from_codes(x_q, s_x, w_q_ref, s_w_ref))
    check_codes(x_q, s_x, np32(x), cfg.group)
    y_ref = O.w8a8_linear(np32(x), w_q_ref, s_w_ref, cfg.group)
    assert _max_rel(np32(y), y_ref) <= 1e-2


@pytest.mark.parametrize("name", ["dit_qkv", "dit_out", "dit_ffn_gate", "dit_ffn_down",
                                  "dit_adaln"])
def test_dense_dit_linear_parity(name):
    """The dense-DiT ConvRot linears at full size (K = 3840 and 10240 take the
    general rotation kernel): weights bit-exact; all activation codes within
    the budget; 64 sampled output rows bit-exact given the GPU's codes and
    within 1e-2 of the oracle's linear."""
    from synthetic import DIT_LINEARS
    cfg = DIT_LINEARS[name]
    x, w = linear_inputs(cfg)
    w_q, s_w = W.convrot_quantize_weights(w.cuda(), cfg.group)
    y, x_q, s_x = _linear_with_codes(x.cuda(), w_q, s_w, cfg.group)
    w_q_ref, s_w_ref = O.rotquant(np32(w), cfg.group)
    assert np.array_equal(w_q.cpu().numpy(), w_q_ref) and np.array_equal(s_w.cpu().numpy(), s_w_ref)
    x_q, s_x = x_q.cpu().numpy(), s_x.cpu().numpy()
    check_codes(x_q, s_x, np32(x), cfg.group)
    rows = np.unique(np.random.default_rng(0).integers(0, cfg.m, 64))
    y_np = np32(y)
    assert np.array_equal(y_np[rows], O.w8a8_linear_from_codes(x_q[rows], s_x[rows], w_q_ref,
                                                                s_w_ref))
    y_ref = O.w8a8_linear(np32(x)[rows], w_q_ref, s_w_ref, cfg.group)
    assert _max_rel(y_np[rows], y_ref) <= 1e-2


@pytest.mark.parametrize("g", [1, 16, 256])
def test_linear_rotation_off_ablation(g):
    """The rotation-off ablation (g = 1: per-token / per-channel INT8 with no
    Hadamard) runs through the same kernels, with the parity of the ConvRot
    linear; on the outlier-laden gate|up inputs the rotation lowers the error
    against the exact product (the reason for ConvRot)."""
    x, w = linear_inputs(LINEAR_CONFIGS["gateup_4096x3072x2048"])
    x, w = x[:256], w[:512]
    w_q, s_w = W.convrot_quantize_weights(w.cuda(), g)
    y, x_q, s_x = _linear_with_codes(x.cuda(), w_q, s_w, g)
    y = np32(y)
    w_q_ref, s_w_ref = O.rotquant(np32(w), g)
    assert np.array_equal(w_q.cpu().numpy(), w_q_ref)
    x_q, s_x = x_q.cpu().numpy(), s_x.cpu().numpy()
    assert np.array_equal(y, O.w8a8_linear_from_codes(x_q, s_x, w_q_ref, s_w_ref))
    check_codes(x_q, s_x, np32(x), g)
    exact = np32(x).astype(np.float64) @ np32(w).astype(np.float64).T
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < {1: 0.06, 16: 0.02, 256: 0.014}[g]
    if g == 1:
        assert rel > 0.03  # without rotation the outlier channels cost accuracy


def test_moe_block_rotation_off():
    """The whole block with g_gu = g_d = 1 (rotation off) against the oracle."""
    base = MOE_CONFIGS["moe_small"]
    cfg = base.__class__(**{**base.__dict__, "g_gu": 1, "g_d": 1})
    inp = moe_inputs(cfg)
    y, v, _ = _run_moe(inp, cfg)
    ow = _oracle_weights(inp, cfg, range(cfg.n_exp))
    y_ref, it = O.moe_block(np32(inp["x"]), np32(inp["logits"]), *ow, c=cfg.c, g_gu=1, g_d=1,
                            keep=True)
    check_codes(v["x_q"].cpu().numpy(), v["s_x"].cpu().numpy(), np32(inp["x"]), 1)
    assert np.array_equal(v["idx"].cpu().numpy(), it["idx"])
    assert _max_rel(np32(y), y_ref) <= 1e-2


def test_linear_empty_batch():
    w = torch.randn(32, 256).to(torch.bfloat16).cuda()
    w_q, s_w = W.convrot_quantize_weights(w, 256)
    y = W.w8a8_convrot_linear(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), w_q, s_w, 256)
    assert y.shape == (0, 32)


# -------------------------------------------------------------- MoE block --
def _quantise_moe_on_gpu(inp, cfg):
    """Tiled weights for the block, plus row-major views of the same codes."""
    gu, dn = W.quantize_moe_weights(inp["wgu"].cuda(), inp["wd"].cuda(), cfg.g_gu, cfg.g_d)
    views = (W.untile(gu).view(cfg.n_exp, 2 * cfg.f, cfg.d), gu.scale.view(cfg.n_exp, 2 * cfg.f),
             W.untile(dn).view(cfg.n_exp, cfg.d, cfg.f), dn.scale.view(cfg.n_exp, cfg.d))
    return (gu, dn), views


def _oracle_weights(inp, cfg, experts):
    e_n, f, d = cfg.n_exp, cfg.f, cfg.d
    wgu_q = np.zeros((e_n, 2 * f, d), np.int8)
    s_gu = np.zeros((e_n, 2 * f), np.float32)
    wd_q = np.zeros((e_n, d, f), np.int8)
    s_d = np.zeros((e_n, d), np.float32)
    for e in experts:
        wgu_q[e], s_gu[e] = O.rotquant(np32(inp["wgu"][e]), cfg.g_gu)
        wd_q[e], s_d[e] = O.rotquant(np32(inp["wd"][e]), cfg.g_d)
    return wgu_q, s_gu, wd_q, s_d


def _run_moe(inp, cfg, t=None):
    t = cfg.t if t is None else t
    (gu, dn), wq = _quantise_moe_on_gpu(inp, cfg)
    ws = torch.empty(W.moe_workspace_size(t, cfg.d, cfg.f, cfg.n_exp, cfg.c), dtype=torch.uint8,
                     device="cuda")
    y = W.moe_expert_choice_forward(inp["x"].cuda(), inp["logits"].cuda(), gu, dn, cfg.c,
                                    cfg.g_gu, cfg.g_d, workspace=ws)
    torch.cuda.synchronize()
    views = W.moe_stage_views(ws, t, cfg.d, cfg.f, cfg.n_exp, cfg.c)
    return y, views, wq


def _max_rel(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _check_block_stages(v, inp, cfg, it, experts, wq_ref):
    """Stage by stage, each GPU stage against the oracle given the GPU's own
    inputs to it: x codes (budget), routing (exact), h codes (budget, from the
    oracle's SwiGLU of the GPU's gathered codes), z (bit-exact given the GPU's
    h codes). Returns the h-code flips and the number of h codes checked."""
    x_q = v["x_q"].cpu().numpy()
    s_x = v["s_x"].cpu().numpy()
    wgu_q, s_gu, wd_q, s_d = wq_ref
    idx = v["idx"].cpu().numpy()
    assert np.array_equal(idx, it["idx"])
    assert np.array_equal(v["w"].cpu().numpy(), it["w"])
    assert np.array_equal(v["x_g"].cpu().numpy(), x_q[idx])
    assert np.array_equal(v["s_g"].cpu().numpy(), s_x[idx])
    flips = codes = 0
    for e in experts:
        rows = idx[e]
        h = O.swiglu_from_codes(x_q[rows], s_x[rows], wgu_q[e], s_gu[e])
        if cfg.g_d == 256:  # stored fp32 h: SwiGLU within CUDA expf's few ulp
            assert _fp32_ulps(v["h"][e].cpu().numpy(), h).max() <= 4
        h_q = v["h_q"][e].cpu().numpy()
        s_h = v["s_h"][e].cpu().numpy()
        n, c, _, _ = check_codes(h_q, s_h, h, cfg.g_d, input_err=8.0)
        flips += n
        codes += c
        z = O.down_from_codes(h_q, s_h, wd_q[e], s_d[e])
        assert np.array_equal(np32(v["z"][e]), z)
    return flips, codes


# g_d = 256 takes the fp32 h + rotation-kernel path (a group of 256 spans
# four epilogue threads); g_d <= 64 rotates and requantises h in the gate/up
# GEMM's epilogue and stores no fp32 h.
_MOE_EXTRA = {
    "moe_small_gd256": MOE_CONFIGS["moe_small_c40"].__class__(
        "moe_small_gd256", 300, 512, 5, 256, 40, 13, g_gu=256, g_d=256),
    "moe_small_gd16": MOE_CONFIGS["moe_small"].__class__(
        "moe_small_gd16", 640, 768, 6, 320, 160, 14, g_gu=64, g_d=16),
}


@pytest.mark.parametrize("name", ["moe_small", "moe_small_c40", "moe_small_gd256",
                                  "moe_small_gd16"])
def test_moe_block_small_end_to_end(name):
    cfg = MOE_CONFIGS[name] if name in MOE_CONFIGS else _MOE_EXTRA[name]
    inp = moe_inputs(cfg)
    y, v, wq = _run_moe(inp, cfg)
    ow = _oracle_weights(inp, cfg, range(cfg.n_exp))
    for got, ref in zip(wq, ow):  # offline weights: bit-exact
        assert np.array_equal(got.cpu().numpy(), ref)
    y_ref, it = O.moe_block(np32(inp["x"]), np32(inp["logits"]), *ow, c=cfg.c, g_gu=cfg.g_gu,
                            g_d=cfg.g_d, keep=True)
    check_codes(v["x_q"].cpu().numpy(), v["s_x"].cpu().numpy(), np32(inp["x"]), cfg.g_gu)
    assert _ulp_diff(v["s_t"].cpu().numpy(), it["scores"].T).max() <= 1
    _check_block_stages(v, inp, cfg, it, range(cfg.n_exp), ow)
    # the combine, bit-exact given the GPU's expert outputs
    z = {e: np32(v["z"][e]) for e in range(cfg.n_exp)}
    y_np = np32(y)
    assert np.array_equal(y_np, O.combine(cfg.t, it["idx"], it["w"], z))
    # and the whole block against the oracle's
    assert _max_rel(y_np, y_ref) <= 1e-2
    unchosen = np.setdiff1d(np.arange(cfg.t), np.unique(it["idx"]))
    assert np.all(y_np[unchosen] == 0)


def test_moe_block_graph_capture_matches_eager():
    """The whole call (with its side-stream routing fork) captured in a CUDA
    graph and replayed on fresh inputs gives the eager result."""
    cfg = MOE_CONFIGS["moe_small"]
    inp = moe_inputs(cfg)
    gu, dn = W.quantize_moe_weights(inp["wgu"].cuda(), inp["wd"].cuda(), cfg.g_gu, cfg.g_d)
    x = inp["x"].cuda()
    logits = inp["logits"].cuda()
    ws = torch.empty(W.moe_workspace_size(cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c), dtype=torch.uint8,
                     device="cuda")
    y = torch.empty(cfg.t, cfg.d, dtype=torch.bfloat16, device="cuda")
    W.moe_expert_choice_forward(x, logits, gu, dn, cfg.c, cfg.g_gu, cfg.g_d, y=y, workspace=ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        W.moe_expert_choice_forward(x, logits, gu, dn, cfg.c, cfg.g_gu, cfg.g_d, y=y, workspace=ws)
    gen = torch.Generator().manual_seed(77)
    x2 = torch.randn(cfg.t, cfg.d, generator=gen).to(torch.bfloat16)
    l2 = torch.randn(cfg.t, cfg.n_exp, generator=gen).to(torch.bfloat16)
    x.copy_(x2.cuda())
    logits.copy_(l2.cuda())
    graph.replay()
    torch.cuda.synchronize()
    y_graph = y.clone()
    y_eager = W.moe_expert_choice_forward(x2.cuda(), l2.cuda(), gu, dn, cfg.c, cfg.g_gu, cfg.g_d)
    torch.cuda.synchronize()
    assert torch.equal(y_graph, y_eager)
    del graph


def test_moe_block_capacity_extremes():
    base = MOE_CONFIGS["moe_small_c40"]
    for c in (0, 1, base.t):
        cfg = base.__class__(**{**base.__dict__, "c": c})
        inp = moe_inputs(cfg)
        y, _, _ = _run_moe(inp, cfg)
        ow = _oracle_weights(inp, cfg, range(cfg.n_exp))
        y_ref = O.moe_block(np32(inp["x"]), np32(inp["logits"]), *ow, c=c, g_gu=cfg.g_gu,
                            g_d=cfg.g_d)
        assert _max_rel(np32(y), y_ref) <= 1e-2 if c > 0 else np.all(np32(y) == 0)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["moe_T8192", "moe_T2048"])
def test_moe_block_full_size(name):
    """The full-size block as the bench runs it, every stage at full size:
    weights bit-exact; all T rows of x codes and all E*C rows of h codes within
    the budget (h from the oracle's SwiGLU of the GPU's gathered codes); routing
    exact; every expert output z bit-exact given the GPU's h codes; every
    output row bit-exact given z; sampled rows within 1e-2 of the oracle's
    whole block."""
    cfg = MOE_CONFIGS[name]
    inp = moe_inputs(cfg)
    y, v, wq = _run_moe(inp, cfg)
    x_np, logits_np = np32(inp["x"]), np32(inp["logits"])
    ow = _oracle_weights(inp, cfg, range(cfg.n_exp))
    for got, ref in zip(wq, ow):
        assert np.array_equal(got.cpu().numpy(), ref)
    idx_ref, w_ref = O.expert_choice_topc(O.router_softmax(logits_np), cfg.c)
    fx, nx, _, _ = check_codes(v["x_q"].cpu().numpy(), v["s_x"].cpu().numpy(), x_np, cfg.g_gu)
    fh, nh = _check_block_stages(v, inp, cfg, {"idx": idx_ref, "w": w_ref}, range(cfg.n_exp), ow)
    print(f"\n{name}: x codes off by one {fx} of {nx} ({fx / nx:.2e}); "
          f"h codes off by one {fh} of {nh} ({fh / nh:.2e})")
    z = {e: np32(v["z"][e]) for e in range(cfg.n_exp)}
    y_np = np32(y)
    assert np.array_equal(y_np, O.combine(cfg.t, idx_ref, w_ref, z))
    counts = np.bincount(idx_ref.ravel(), minlength=cfg.t)
    rng = np.random.default_rng(0)
    busy = np.argsort(-counts, kind="stable")[:8]
    sample = np.unique(np.concatenate([np.arange(8), rng.choice(cfg.t, 16, replace=False), busy]))
    y_ref = O.moe_block(x_np, logits_np, *ow, c=cfg.c, g_gu=cfg.g_gu, g_d=cfg.g_d,
                        out_tokens=sample)
    assert _max_rel(y_np[sample], y_ref[sample]) <= 1e-2


# ---------------------------------------------------------- failure path --
def test_bounded_wait_gives_up_and_reports():
    assert W.convrot_wait_selftest(2_000_000) == 0   # 2 ms limit, nothing arrives
    flags = W.convrot_check_device_error()
    assert flags & (1 << 5)
    assert W.convrot_check_device_error() == 0       # cleared by the read


def test_cross_tile_wait_gives_up_and_reports():
    """The bounded counter wait between the requantising GEMM's tiles, on a
    counter nothing raises: it gives up after its limit and the host reads
    CONVROT_ERR_TIMEOUT (the self-test bit); the context stays usable."""
    assert W.convrot_count_wait_selftest(2_000_000) == 0   # 2 ms limit
    flags = W.convrot_check_device_error()
    assert flags & (1 << 5)
    assert W.convrot_check_device_error() == 0
    # the device still runs work afterwards
    q, s = W.convrot_rotquant(torch.ones(4, 256, dtype=torch.bfloat16, device="cuda"), 256)
    assert float(s[0]) > 0
