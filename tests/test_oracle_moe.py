"""Pins for the oracle's router, expert-choice top-C and MoE block (no GPU).

Definitions: "MLX Nucleus-Image", opening paragraph (64 routed experts with
expert-choice routing) and table "Conversion notes" (each expert picks its
top-C tokens, outputs scattered back; experts compute silu(gate) * up with
gate in the first half); "Nucleus-Image INT8 Convrot Experts + FP8 Text
Encoder", section "Quantization" (group 256 for gate/up, 64 for down).
"""

import numpy as np
import pytest
import scipy.special
import torch

from oracle import (bf16_round, expert_choice_topc, moe_block, rotquant,
                    router_softmax, silu_f32)
from tests.golden import read_fixture


def test_softmax_matches_library(rng):
    logits = torch.from_numpy(rng.standard_normal((200, 64)).astype(np.float32))
    logits = logits.to(torch.bfloat16).float().numpy()
    s = router_softmax(logits)
    ref = scipy.special.softmax(logits.astype(np.float64), axis=1)
    ulp = np.spacing(ref.astype(np.float32))
    assert s.dtype == np.float32
    assert np.all(np.abs(s.astype(np.float64) - ref) <= ulp)
    assert np.allclose(s.sum(1), 1.0, atol=64 * 2.0 ** -24)


def test_softmax_closed_forms():
    s = router_softmax(np.zeros((1, 64), np.float32))
    assert np.all(s == np.float32(1 / 64))
    s = router_softmax(np.array([[0.0, -200.0], [3.0, 3.0]], np.float32))
    assert s.tolist() == [[1.0, 0.0], [0.5, 0.5]]
    # large logits (bf16 reaches 3e38): the max is taken out before exp
    s = router_softmax(np.array([[1000.0, 1000.0, -1000.0]], np.float32))
    assert s.tolist() == [[0.5, 0.5, 0.0]]


def _topc_brute(scores, c):
    t, e_n = scores.shape
    idx = []
    for e in range(e_n):
        order = sorted(range(t), key=lambda i: (-float(scores[i, e]), i))
        idx.append(sorted(order[:c]))
    return np.array(idx, dtype=np.int32).reshape(e_n, c)


@pytest.mark.parametrize("t,c", [(1, 1), (17, 5), (64, 64), (100, 0), (257, 13)])
def test_topc_brute_force(t, c, rng):
    # coarse scores force many exact ties
    scores = (rng.integers(0, 7, size=(t, 4)) / 8).astype(np.float32)
    idx, w = expert_choice_topc(scores, c)
    assert np.array_equal(idx, _topc_brute(scores, c))
    for e in range(4):
        assert len(set(idx[e].tolist())) == c
        assert np.all(np.diff(idx[e]) > 0)
        assert np.array_equal(w[e], scores[idx[e], e])


def test_silu_closed_forms():
    g = np.array([0.0, 127.0, -16129.0, 20.0, -1.0], np.float32)
    h = silu_f32(g)
    assert h[0] == 0.0 and h[1] == 127.0 and h[2] == 0.0 and np.signbit(h[2])
    assert h[3] == np.float32(20.0)  # 1 + exp(-20) rounds to 1 in fp32
    assert abs(h[4] - (-1.0 / (1.0 + np.e))) < 1e-7


def _rows(fx, key):
    return np.array(fx[key], dtype=np.float64)


def test_worked_moe_block():
    fx = read_fixture("moe_tiny_worked.txt")
    x = _rows(fx, "x").astype(np.float32)
    logits = _rows(fx, "logits").astype(np.float32)
    wgu = np.stack([_rows(fx, "wgu0"), _rows(fx, "wgu1")])
    wd = np.stack([_rows(fx, "wd0"), _rows(fx, "wd1")])
    wgu_q = np.zeros(wgu.shape, np.int8)
    s_gu = np.zeros(wgu.shape[:2], np.float32)
    wd_q = np.zeros(wd.shape, np.int8)
    s_d = np.zeros(wd.shape[:2], np.float32)
    for e in range(2):
        wgu_q[e], s_gu[e] = rotquant(wgu[e], 1)
        wd_q[e], s_d[e] = rotquant(wd[e], 1)
    assert np.all(s_gu == 1) and np.all(s_d == 1)
    y, inter = moe_block(x, logits, wgu_q, s_gu, wd_q, s_d, c=2, g_gu=1, g_d=1, keep=True)
    assert inter["idx"].tolist() == fx["idx"]
    assert inter["w"].tolist() == fx["w"]
    assert inter["out32"].tolist() == fx["out32"]
    assert y.tolist() == fx["y"]


def _quantise_block_weights(wgu, wd, g_gu, g_d):
    e_n = wgu.shape[0]
    wgu_q = np.zeros(wgu.shape, np.int8)
    s_gu = np.zeros(wgu.shape[:2], np.float32)
    wd_q = np.zeros(wd.shape, np.int8)
    s_d = np.zeros(wd.shape[:2], np.float32)
    for e in range(e_n):
        wgu_q[e], s_gu[e] = rotquant(wgu[e], g_gu)
        wd_q[e], s_d[e] = rotquant(wd[e], g_d)
    return wgu_q, s_gu, wd_q, s_d


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def test_single_dense_expert_is_a_swiglu_mlp(rng):
    """E = 1, C = T: every router weight is 1 and the block is a dense MLP."""
    t, d, f = 48, 512, 192
    x = _bf16(rng.standard_normal((t, d)))
    logits = _bf16(rng.standard_normal((t, 1)))
    wgu = _bf16(rng.standard_normal((1, 2 * f, d)) * 0.02)
    wd = _bf16(rng.standard_normal((1, d, f)) * 0.02)
    q = _quantise_block_weights(wgu, wd, 256, 64)
    y, inter = moe_block(x, logits, *q, c=t, keep=True)
    assert np.all(inter["w"] == 1.0)
    x64 = x.astype(np.float64)
    gate = x64 @ wgu[0, :f].T
    up = x64 @ wgu[0, f:].T
    h = gate / (1 + np.exp(-gate)) * up
    ref = h @ wd[0].astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.03
    # swapping the halves (silu(up) * gate) is far off: the order is pinned
    h_sw = up / (1 + np.exp(-up)) * gate
    assert np.linalg.norm(h_sw @ wd[0].astype(np.float64).T - ref) / np.linalg.norm(ref) > 0.3


def test_block_against_unquantised_block(rng):
    """Same routing, fp64 unquantised experts: the INT8 error stays small."""
    t, d, e_n, f, c = 96, 512, 4, 128, 40
    x = _bf16(rng.standard_normal((t, d)))
    logits = _bf16(rng.standard_normal((t, e_n)))
    wgu = _bf16(rng.standard_normal((e_n, 2 * f, d)) * 0.02)
    wd = _bf16(rng.standard_normal((e_n, d, f)) * 0.02)
    q = _quantise_block_weights(wgu, wd, 256, 64)
    y, inter = moe_block(x, logits, *q, c=c, keep=True)
    ref = np.zeros((t, d))
    for e in range(e_n):
        rows = inter["idx"][e]
        xe = x[rows].astype(np.float64)
        gate, up = xe @ wgu[e, :f].T, xe @ wgu[e, f:].T
        ref[rows] += inter["w"][e][:, None] * ((gate / (1 + np.exp(-gate)) * up) @ wd[e].T)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.03
    unchosen = np.setdiff1d(np.arange(t), np.unique(inter["idx"]))
    assert np.all(y[unchosen] == 0)
    assert np.array_equal(y, bf16_round(inter["out32"]))


def test_int32_accumulator_bound_at_block_sizes():
    """K * 127^2 < 2^31 for K = d = 2048 and K = f = 1536."""
    assert 2048 * 127 * 127 < 2**31 and 1536 * 127 * 127 < 2**31


def test_down_rotation_group_is_local(rng):
    """h is rotated in groups of g_d = 64 along f: an h row that is zero
    beyond column 64 keeps all-zero codes there (a 256 group would spread)."""
    t, d, f = 16, 256, 256
    x = _bf16(rng.standard_normal((t, d)))
    logits = _bf16(rng.standard_normal((t, 1)))
    wgu = _bf16(rng.standard_normal((1, 2 * f, d)) * 0.02)
    wgu[0, 64:f] = 0.0          # gate columns 64.. are zero -> h[:, 64:] = 0
    wd = _bf16(rng.standard_normal((1, d, f)) * 0.02)
    q = _quantise_block_weights(wgu, wd, 256, 64)
    _, inter = moe_block(x, logits, *q, c=t, g_gu=256, g_d=64, keep=True)
    hq = inter["h_q"][0]
    assert np.all(inter["h"][0][:, 64:] == 0)
    assert np.all(hq[:, 64:] == 0) and np.all(np.abs(hq[:, :64]).max(1) == 127)
