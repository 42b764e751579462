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


def test_gemm_roofline_bytes_are_weights_and_scales():
    """The roofline of a GEMM counts its weights once plus their scales; the
    gathered activation codes and the h codes are not algorithmic traffic."""
    cfg = MOE_CONFIGS["moe_T8192"]
    w = bench.algorithmic_work(cfg, cfg.t)
    assert w["gateup_alg"]["bytes"] == 402_653_184 + 786_432
    assert w["down_alg"]["bytes"] == 201_326_592 + 524_288
    assert w["gateup_alg"]["ops"] == w["gateup"]["ops"]


def test_roofline_fractions():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 500.0}  # int8 peak = 1000 TOPS
    r = bench.roofline_of(ops=2e12, nbytes=1e9, seconds=4e-3, peaks=peaks)
    assert r["bound"] == "tensor"                      # 2 ms of tensor work > 1 ms of HBM
    assert abs(r["hbm_gbs"] - 250.0) < 1e-9 and abs(r["hbm_frac"] - 0.25) < 1e-12
    assert abs(r["tops"] - 500.0) < 1e-9 and abs(r["tensor_frac"] - 0.5) < 1e-12
    assert abs(r["roofline_frac"] - 0.5) < 1e-12 and abs(r["ideal_us"] - 2000.0) < 1e-6


def test_traffic_record_needs_the_current_sources(tmp_path, monkeypatch):
    """A traffic figure counts only while the kernel sources are those it was
    captured on."""
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    (tmp_path / "k.md").write_text(
        "# summary\ntraffic-record: kernel=gemm_x workload=moe_T8192 bytes_per_launch=4.5e8 "
        f"source_sha16={bench.source_sha16()}\n"
        "traffic-record: kernel=gemm_y workload=moe_T8192 bytes_per_launch=1e8 "
        "source_sha16=0000000000000000\n")
    assert bench.profile_traffic("gemm_x", "moe_T8192")[0] == 4.5e8
    got, note = bench.profile_traffic("gemm_y", "moe_T8192")
    assert got is None and "changed" in note
    assert bench.profile_traffic("gemm_x", "moe_T2048")[0] is None


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    """The hash that keys the traffic records changes with the code of the
    CUDA sources or the header, not with their comments or blank lines."""
    csrc = tmp_path / "w8a8_rotated_int8_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "include").mkdir()
    kern = csrc / "k.cuh"
    head = tmp_path / "include" / "convrot.h"
    kern.write_text("// a kernel\n__global__ void k(int* p) { p[0] = 1; }\n")
    head.write_text("/* the ABI */\nint f(void);\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.source_sha16()
    kern.write_text("// a kernel, now documented\n\n__global__ void k(int* p) { p[0] = 1; }  // one\n")
    head.write_text("/* the ABI,\n   in two lines */\nint f(void);  /* f */\n")
    assert bench.source_sha16() == base
    kern.write_text("// a kernel\n__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.source_sha16() != base


class _FakeNvml:
    """Stands in for pynvml: the SM clock and reasons change with a phase the
    test sets (before, during and after the timed region)."""

    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    def __init__(self):
        self.phase = "before"

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return 1965 if self.phase == "during" else 900

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.nvmlClocksEventReasonSwPowerCap if self.phase == "during" else \
            self.nvmlClocksEventReasonHwSlowdown


def test_clock_sampler_reports_only_the_timed_window():
    """Samples taken before begin() or after end() (here: a slow clock and a
    hardware slowdown) stay out of the record; the window's samples give the
    median clock and the reasons active in it."""
    import time
    nv = _FakeNvml()
    clk = bench.ClockSampler(None, nvml=nv)
    clk.start()
    assert clk.samples, "the sampler is warm when start() returns"
    time.sleep(0.02)
    nv.phase = "during"
    time.sleep(0.002)
    clk.begin()
    time.sleep(0.03)
    clk.end()
    time.sleep(0.002)
    nv.phase = "after"
    time.sleep(0.02)
    rec = clk.stop()
    assert rec["sm_mhz"] == 1965 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] >= 10


def test_clock_sampler_without_nvml():
    class Broken:
        def nvmlInit(self):
            raise RuntimeError("no driver")
    clk = bench.ClockSampler(None, nvml=Broken())
    clk.start()
    clk.begin()
    clk.end()
    assert clk.stop()["reasons"] == ["nvml unavailable"]
