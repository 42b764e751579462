"""Workload recipes: shapes, distributions and seeds of the synthetic inputs.

The pages measure on real prompts, images and trained weights that are not
available here; these seeded tensors stand in for them with the shapes and
value distributions of the workloads (activations N(0,1) with 1% of the
K-channels scaled by 20 as outliers, weights N(0,0.02), router logits N(0,1)).

All tensors are drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in fp32 and cast to bf16 (round to nearest even). Draw order within a seed is
fixed: activations, outlier channels, logits, gate/up weights expert by
expert, down weights expert by expert.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearConfig:
    name: str
    m: int
    n: int
    k: int
    group: int
    seed: int
    swiglu_input: bool = False  # X = bf16(silu(gate) * up) from bf16 gate/up


@dataclass(frozen=True)
class MoEConfig:
    name: str
    t: int
    d: int
    n_exp: int
    f: int
    c: int
    seed: int
    g_gu: int = 256
    g_d: int = 64


LINEAR_CONFIGS = {
    # single ConvRot linear, 64 tokens, K = N = 256, one rotation group
    "linear_64x256x256": LinearConfig("linear_64x256x256", 64, 256, 256, 256, 0),
    # fused gate|up projection of a 4096-token batch
    "gateup_4096x3072x2048": LinearConfig("gateup_4096x3072x2048", 4096, 3072, 2048, 256, 1),
    # down projection, input from a SwiGLU of seeded gate/up
    "down_4096x2048x1536": LinearConfig("down_4096x2048x1536", 4096, 2048, 1536, 64, 2,
                                        swiglu_input=True),
}

# The dense-DiT W8A8 ConvRot linears of one transformer block (the int8
# ConvRot files of "NitroFusion2 for ComfyUI: int8, W6A8, W4A8", section "How
# they were made": all linears of the main and refiner blocks -- attention qkv
# and out, the three feed-forward layers, adaLN -- with a block Hadamard of
# 256). The page gives 202 linears and 6.142B quantised weights, not their
# shapes; assumed here: 34 blocks of six linears, hidden size 3840, a SwiGLU
# feed-forward of 10240 and an adaLN projection of a 256-wide conditioning
# vector to four modulation vectors, which gives 6.15B weights. Tokens: a
# 1024x1024 image as 4096 tokens (the one-step model runs without CFG); the
# adaLN input is one row per image.
DIT_D, DIT_F = 3840, 10240
DIT_LINEARS = {
    "dit_qkv": LinearConfig("dit_qkv", 4096, 3 * DIT_D, DIT_D, 256, 21),
    "dit_out": LinearConfig("dit_out", 4096, DIT_D, DIT_D, 256, 22),
    "dit_ffn_gate": LinearConfig("dit_ffn_gate", 4096, DIT_F, DIT_D, 256, 23),
    "dit_ffn_up": LinearConfig("dit_ffn_up", 4096, DIT_F, DIT_D, 256, 24),
    "dit_ffn_down": LinearConfig("dit_ffn_down", 4096, DIT_D, DIT_F, 256, 25, swiglu_input=True),
    "dit_adaln": LinearConfig("dit_adaln", 1, 4 * DIT_D, 256, 256, 26),
}

MOE_CONFIGS = {
    # 1024x1024 image with batched CFG: 8192 tokens, capacity factor 2
    "moe_T8192": MoEConfig("moe_T8192", 8192, 2048, 64, 1536, 256, 3),
    # 512x512 image with batched CFG: the weight-bound small-batch regime
    "moe_T2048": MoEConfig("moe_T2048", 2048, 2048, 64, 1536, 64, 4),
    # token sweep of the same block, C = 2T/64
    "moe_T512": MoEConfig("moe_T512", 512, 2048, 64, 1536, 16, 5),
    "moe_T1024": MoEConfig("moe_T1024", 1024, 2048, 64, 1536, 32, 6),
    "moe_T4096": MoEConfig("moe_T4096", 4096, 2048, 64, 1536, 128, 7),
    # oracle-sized blocks: several tiles plus ragged tails in every dimension
    "moe_small": MoEConfig("moe_small", 640, 768, 6, 320, 160, 11),
    "moe_small_c40": MoEConfig("moe_small_c40", 300, 512, 5, 192, 40, 12),
}


def outlier_channels(k: int, gen: torch.Generator) -> torch.Tensor:
    """1% of the K channels (at least one), drawn without replacement."""
    n = max(1, int(round(0.01 * k)))
    return torch.randperm(k, generator=gen)[:n]


def _activations(rows: int, k: int, gen: torch.Generator, outliers: bool = True) -> torch.Tensor:
    x = torch.randn(rows, k, generator=gen, dtype=torch.float32)
    if outliers:
        ch = outlier_channels(k, gen)
        x[:, ch] *= 20.0
    return x.to(torch.bfloat16)


def _weights(rows: int, k: int, gen: torch.Generator) -> torch.Tensor:
    return (torch.randn(rows, k, generator=gen, dtype=torch.float32) * 0.02).to(torch.bfloat16)


def linear_inputs(cfg: LinearConfig):
    """Returns (X bf16 [M, K], W bf16 [N, K]) on the CPU."""
    gen = torch.Generator().manual_seed(cfg.seed)
    if cfg.swiglu_input:
        gate = torch.randn(cfg.m, cfg.k, generator=gen, dtype=torch.float32).to(torch.bfloat16)
        up = torch.randn(cfg.m, cfg.k, generator=gen, dtype=torch.float32).to(torch.bfloat16)
        # input synthesis only: the down projection sees a SwiGLU-shaped input
        x = (torch.nn.functional.silu(gate.float()) * up.float()).to(torch.bfloat16)
    else:
        x = _activations(cfg.m, cfg.k, gen)
    w = _weights(cfg.n, cfg.k, gen)
    return x, w


def moe_inputs(cfg: MoEConfig, t: int | None = None, weights: bool = True):
    """Returns dict of CPU tensors: x [T,d], logits [T,E] (bf16),
    wgu [E,2f,d] (bf16; rows 0..f-1 gate, f..2f-1 up), wd [E,d,f] (bf16).

    ``t`` overrides the token count (the weights do not depend on it);
    ``weights=False`` draws only x and the logits (the same values).
    """
    t = cfg.t if t is None else t
    gen = torch.Generator().manual_seed(cfg.seed)
    x = _activations(t, cfg.d, gen)
    logits = torch.randn(t, cfg.n_exp, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    if not weights:
        return {"x": x, "logits": logits}
    wgu = torch.empty(cfg.n_exp, 2 * cfg.f, cfg.d, dtype=torch.bfloat16)
    for e in range(cfg.n_exp):
        wgu[e] = _weights(2 * cfg.f, cfg.d, gen)
    wd = torch.empty(cfg.n_exp, cfg.d, cfg.f, dtype=torch.bfloat16)
    for e in range(cfg.n_exp):
        wd[e] = _weights(cfg.d, cfg.f, gen)
    return {"x": x, "logits": logits, "wgu": wgu, "wd": wd}
