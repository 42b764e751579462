"""Pins for the oracle's block-Hadamard rotation (no GPU).

Definition: "Nucleus-Image INT8 Convrot Experts + FP8 Text Encoder",
section "Quantization" (ConvRot in groups of 256 / 64 along K) and
"NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How they were made"
(block Hadamard rotation).
"""

from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

from oracle import block_rotate, hadamard, rotation_matrix
from tests.golden import read_fixture


def test_small_hadamards_by_hand():
    assert hadamard(1).tolist() == [[1]]
    assert hadamard(2).tolist() == [[1, 1], [1, -1]]
    assert hadamard(4).tolist() == [[1, 1, 1, 1], [1, -1, 1, -1],
                                    [1, 1, -1, -1], [1, -1, -1, 1]]


@pytest.mark.parametrize("g", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_orthogonality_exact(g):
    h = hadamard(g)
    assert np.array_equal(h @ h.T, g * np.eye(g, dtype=np.int64))
    assert np.array_equal(h, h.T)


@pytest.mark.parametrize("g", [2, 4, 16, 64, 256])
def test_matches_library_sylvester(g):
    assert np.array_equal(hadamard(g), scipy.linalg.hadamard(g))


@pytest.mark.parametrize("g", [1, 4, 16, 64, 256])
def test_rotation_orthonormal(g):
    r = rotation_matrix(g)
    assert np.allclose(r @ r.T, np.eye(g), atol=1e-14, rtol=0)
    # 1/sqrt(g) is a power of two for powers of four: entries are exact
    assert set(np.unique(np.abs(r))) == {1.0 / np.sqrt(g)}


def test_rejects_non_power_of_four():
    for g in (2, 8, 32, 128, 3):
        with pytest.raises(ValueError):
            rotation_matrix(g)


def test_worked_rotation_g4():
    fx = read_fixture("rotation_g4.txt")
    v = np.array(fx["input"][0])
    assert block_rotate(v[None, :], 4)[0].tolist() == fx["rotated"][0]


def test_rotation_g1_is_identity(rng):
    x = rng.standard_normal((3, 32))
    assert np.array_equal(block_rotate(x, 1), x)


def test_block_locality_and_rows():
    k, g = 512, 256
    r = rotation_matrix(g)
    for j in (0, 37, 255, 256, 300, 511):
        e = np.zeros((1, k))
        e[0, j] = 1.0
        out = block_rotate(e, g)[0]
        blk = j // g
        expect = np.zeros(k)
        expect[blk * g:(blk + 1) * g] = r[j % g]
        assert np.array_equal(out, expect)


def _fwht_rows(v, g):
    """Independent in-place fast Walsh-Hadamard butterflies per block."""
    v = v.astype(np.float64).copy()
    k = v.shape[-1]
    for base in range(0, k, g):
        span = 1
        while span < g:
            for start in range(base, base + g, 2 * span):
                a = v[..., start:start + span].copy()
                b = v[..., start + span:start + 2 * span].copy()
                v[..., start:start + span] = a + b
                v[..., start + span:start + 2 * span] = a - b
            span *= 2
    return v / np.sqrt(g)


@pytest.mark.parametrize("g", [4, 16, 64, 256])
def test_matches_fast_walsh_hadamard(g, rng):
    import torch
    v = torch.from_numpy(rng.standard_normal((3, 512)).astype(np.float32))
    v = v.to(torch.bfloat16).float().numpy()  # bf16 data: both sides exact
    assert np.array_equal(block_rotate(v, g), _fwht_rows(v, g))


@pytest.mark.parametrize("g", [64, 256])
def test_rotation_invariance_of_product(g, rng):
    x = rng.standard_normal((8, 1024))
    w = rng.standard_normal((6, 1024)) * 0.02
    ref = x @ w.T
    rot = block_rotate(x, g) @ block_rotate(w, g).T
    assert np.max(np.abs(rot - ref)) <= 1e-9 * np.max(np.abs(ref))


def test_rotation_of_bf16_rows_is_exact(rng):
    """bf16 inputs (8-bit significands) rotate exactly in fp64 (g=64)."""
    import torch
    v = torch.from_numpy(rng.standard_normal((2, 64)).astype(np.float32) * 3)
    v = v.to(torch.bfloat16).float().numpy()
    got = block_rotate(v, 64)
    h = hadamard(64)
    for i in range(2):
        exact = [sum(Fraction(float(v[i, k])) * int(h[k, j]) for k in range(64)) / 8
                 for j in range(64)]
        assert [Fraction(float(x)) for x in got[i]] == exact
