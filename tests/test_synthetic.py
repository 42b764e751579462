"""The seeded input generators: shapes, dtypes, determinism (no GPU)."""

import torch

from synthetic import LINEAR_CONFIGS, MOE_CONFIGS, linear_inputs, moe_inputs, outlier_channels


def test_linear_small_shapes_and_determinism():
    cfg = LINEAR_CONFIGS["linear_64x256x256"]
    x, w = linear_inputs(cfg)
    x2, w2 = linear_inputs(cfg)
    assert x.shape == (64, 256) and w.shape == (256, 256)
    assert x.dtype == torch.bfloat16 and w.dtype == torch.bfloat16
    assert torch.equal(x, x2) and torch.equal(w, w2)
    # 3 outlier channels (1% of 256) scaled by 20: their column std is large
    std = x.float().std(0)
    assert int((std > 8).sum()) == 3


def test_outlier_count():
    g = torch.Generator().manual_seed(0)
    assert len(outlier_channels(2048, g)) == 20
    assert len(set(outlier_channels(2048, g).tolist())) == 20


def test_moe_small_shapes():
    cfg = MOE_CONFIGS["moe_small"]
    inp = moe_inputs(cfg)
    assert inp["x"].shape == (cfg.t, cfg.d)
    assert inp["logits"].shape == (cfg.t, cfg.n_exp)
    assert inp["wgu"].shape == (cfg.n_exp, 2 * cfg.f, cfg.d)
    assert inp["wd"].shape == (cfg.n_exp, cfg.d, cfg.f)
    assert abs(float(inp["wgu"].float().std()) - 0.02) < 0.002


def test_dense_dit_block_matches_the_pages_weight_count():
    """The assumed dense-DiT block: 34 blocks of its six linears hold the
    6.142B quantised weights of the NitroFusion2 int8 files within 0.2%, and
    every K is a multiple of the rotation group 256."""
    from synthetic import DIT_LINEARS
    per_block = sum(c.n * c.k for c in DIT_LINEARS.values())
    assert abs(34 * per_block / 6.142e9 - 1) < 2e-3
    assert len(DIT_LINEARS) * 34 == 204  # the page counts 202 quantised linears
    for c in DIT_LINEARS.values():
        assert c.k % 256 == 0 and c.group == 256
