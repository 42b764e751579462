"""bench.py's algorithmic work: the ops and compulsory bytes behind the roofline
figures, checked against the sizes of the workload (no GPU).

At T=8192, d=2048, f=1536, E=64, C=256:
- the expert weights are 64 x (3072 x 2048 + 2048 x 1536) int8 codes (603.98 MB) with one fp32 scale per row
  (1.31 MB);
- the gate/up GEMM is 2 x 64 x 256 x 2048 x 3072 ops (206.2 GOP) and the down GEMM half that (103.1 GOP);
- the block reads X (bf16) and the logits (bf16) and writes Y (bf16).
"""

import bench
from synthetic import MOE_CONFIGS


def test_block_work_at_t8192():
    cfg = MOE_CONFIGS["moe_T8192"]
    w = bench.algorithmic_work(cfg, cfg.t)
    weight_codes = 603_979_776
    weight_scales = 1_310_720
    x_in, logits_in, y_out = 8192 * 2048 * 2, 8192 * 64 * 2, 8192 * 2048 * 2
    assert w["block_bytes"] == weight_codes + weight_scales + x_in + logits_in + y_out
    assert w["gateup"]["ops"] == 206_158_430_208
    assert w["down"]["ops"] == 103_079_215_104
    assert w["ops"] == w["gateup"]["ops"] + w["down"]["ops"]


def test_requantising_gemm_bytes():
    # weights 402.65 MB + scales 0.79 MB + gathered codes and scales in + h codes and scales out
    for name, gathered_rows, expect in (("moe_T8192", 64 * 256, 462_290_944),
                                        ("moe_T2048", 64 * 64, 418_152_448)):
        cfg = MOE_CONFIGS[name]
        w = bench.algorithmic_work(cfg, cfg.t)
        assert w["gateup_rq"]["bytes"] == (402_653_184 + 786_432 + gathered_rows * (2048 + 4)
                                           + gathered_rows * (1536 + 4)) == expect
        # the two-step form writes h as fp32 instead of codes and scales
        assert w["gateup"]["bytes"] - w["gateup_rq"]["bytes"] == gathered_rows * (1536 * 4 - 1540)


def test_fused_h_follows_the_down_group():
    assert bench.fused_h(MOE_CONFIGS["moe_T8192"])
    assert bench.fused_h(MOE_CONFIGS["moe_T2048"])
