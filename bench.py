"""Benchmark of the W8A8 ConvRot expert-choice MoE block on B200.

One step = one pass of the whole hot path (router softmax, activation
rotate+quantise, expert-choice top-C, gather, gate/up GEMM + SwiGLU with the
h rotate+requantise in its epilogue, down GEMM to bf16, router-weighted
combine) over one batch of synthetic tokens, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config moe_T8192]
                    [--impl ours|reference] [--no-cpu-baseline] [--no-extras]
                    [--ablation] [--sweep]

The JSON line reports the configured block (default T=8192), and under
"workloads" the same block at T=2048 (the weight-bound regime, with its
fraction of HBM bandwidth) and at every T of the 512..8192 sweep, the single
W8A8 ConvRot linears (gate|up 4096x3072x2048, down 4096x2048x1536, and
64x256x256) with their fraction of the INT8 tensor peak, the six linears of
one dense-DiT block (4096 tokens, hidden 3840, feed-forward 10240, all with
the 256-group rotation), and a dense INT8 GEMM probe of the tensor peak this
library's own kernel reaches.

Multi-GPU (launched by torch.distributed.run): every rank runs its own batch
of T tokens against the same weights (weak scaling, no data-path
collective); the barrier and the max-over-ranks timing use the process group.
`--impl reference` times the CPU oracle (the only reference there is) on a
bounded sample of the same workload. `--ablation` measures, instead of
throughput, the block's error with ConvRot and with the rotation off.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import (DIT_LINEARS, LINEAR_CONFIGS, MOE_CONFIGS, linear_inputs,  # noqa: E402
                       moe_inputs)

METRIC = "W8A8 ConvRot MoE block tokens/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
INT8_DATASHEET_TOPS = 4500.0  # B200 dense INT8, nominal (context only)
PROFILES = os.path.join(ROOT, "profiles")


def source_sha16():
    """Hash of the CUDA sources and the ABI header without their comments and
    blank lines: a traffic figure captured by ncu on other code no longer
    describes the kernel (a comment does not change it)."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w8a8_rotated_int8_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for path in files + [os.path.join(ROOT, "include", "convrot.h")]:
        with open(path) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profile_traffic(kernel, workload):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of `kernel` on
    `workload`, from a record line of a summary under profiles/:
        traffic-record: kernel=<k> workload=<w> bytes_per_launch=<n> source_sha16=<h>
    Returns (bytes or None, note)."""
    if not os.path.isdir(PROFILES):
        return None, "no profiles directory"
    sha = source_sha16()
    found = None
    for name in sorted(os.listdir(PROFILES)):
        with open(os.path.join(PROFILES, name)) as fh:
            for line in fh:
                if not line.startswith("traffic-record:"):
                    continue
                kv = dict(part.split("=", 1) for part in line.split()[1:] if "=" in part)
                if kv.get("kernel") == kernel and kv.get("workload") == workload:
                    found = (float(kv["bytes_per_launch"]), kv.get("source_sha16"), name)
    if found is None:
        return None, "no ncu capture of this kernel on this workload"
    if found[1] != sha:
        return None, f"kernel sources changed since the capture in profiles/{found[2]}"
    return found[0], f"ncu capture, profiles/{found[2]}"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def algorithmic_work(cfg, t):
    """Ops and compulsory bytes of one block call and of its two GEMM launches.

    The roofline bytes of a GEMM (``*_alg``) are its weights once plus their
    scales: gathered and intermediate copies are not algorithmic traffic.
    ``gateup``/``gateup_rq``/``down`` also count what the launch reads and
    writes of its activations (as-built bytes, for context)."""
    e, c, d, f = cfg.n_exp, cfg.c, cfg.d, cfg.f
    w_bytes = e * (2 * f * d + d * f)
    s_bytes = e * (2 * f + d) * 4
    block_bytes = w_bytes + s_bytes + t * d * 2 + t * e * 2 + t * d * 2
    ops = 2 * e * c * (d * 2 * f + f * d)
    gateup = {
        "ops": 2 * e * c * d * 2 * f,
        # weights + their scales + gathered codes and scales in + h (fp32) out
        "bytes": e * 2 * f * d + e * 2 * f * 4 + e * c * (d + 4) + e * c * f * 4,
    }
    gateup_rq = {
        "ops": 2 * e * c * d * 2 * f,
        # the same inputs; out: h codes and their scales (h stays on chip)
        "bytes": e * 2 * f * d + e * 2 * f * 4 + e * c * (d + 4) + e * c * (f + 4),
    }
    down = {
        "ops": 2 * e * c * f * d,
        # weights + scales + h codes and scales in + bf16 rows out
        "bytes": e * d * f + e * d * 4 + e * c * (f + 4) + e * c * d * 2,
    }
    gateup_alg = {"ops": gateup["ops"], "bytes": e * 2 * f * d + e * 2 * f * 4}
    down_alg = {"ops": down["ops"], "bytes": e * d * f + e * d * 4}
    return {"ops": ops, "block_bytes": block_bytes, "gateup": gateup, "gateup_rq": gateup_rq,
            "down": down, "gateup_alg": gateup_alg, "down_alg": down_alg}


def roofline_of(ops, nbytes, seconds, peaks):
    """Both fractions of one launch (or call): achieved bytes/s against the
    measured HBM copy bandwidth and ops/s against the INT8 tensor peak (2 x
    the measured bf16 burst, the nominal int8:bf16 ratio); the bound is the
    larger of the two ideal times."""
    int8 = 2.0 * peaks["bf16_tflops"]
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = ops / (int8 * 1e12)
    gbs = nbytes / seconds / 1e9
    tops = ops / seconds / 1e12
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor",
            "ideal_us": max(t_hbm, t_tc) * 1e6, "roofline_frac": max(t_hbm, t_tc) / seconds,
            "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
            "tops": tops, "tensor_frac": tops / int8, "tensor_frac_datasheet": tops / INT8_DATASHEET_TOPS}


def fused_h(cfg):
    """Whether the block requantises h in the gate/up GEMM's epilogue (the
    library does for g_d <= 64 on a full B200)."""
    return cfg.g_d <= 64


class ClockSampler:
    """SM clock and clock-event reasons sampled (read-only, NVML) by a thread
    as fast as NVML answers (two queries per sample). The thread starts before
    the timed region, so it is already sampling when the region begins; only
    the samples taken between begin() and end() are reported. `nvml` replaces
    the pynvml module (a fake, for tests without a GPU)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, torch_device, nvml=None):
        import threading
        self.dev = torch_device
        self.samples = []          # (perf_counter seconds, SM MHz, reason bits)
        self.stop_evt = threading.Event()
        self.thread = None
        self.nvml = None
        self.fake = nvml
        self.handle = None
        self.max_mhz = None
        self.window = [None, None]

    def _open(self):
        if self.fake is not None:
            nv = self.fake
            nv.nvmlInit()
            self.handle = nv.nvmlDeviceGetHandleByIndex(0)
        else:
            import pynvml as nv
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.handle = nv.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
        self.nvml = nv

    def _loop(self):
        nv = self.nvml
        while not self.stop_evt.is_set():
            try:
                t = time.perf_counter()
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((t, mhz, rs))
            except Exception:  # noqa: BLE001 - sampling is best effort
                pass
            self.stop_evt.wait(0.0001)

    def start(self):
        """Opens NVML and starts sampling; returns once the first sample is in
        (at most 1 s), so the thread is warm when the timed region begins."""
        import threading
        try:
            self._open()
        except Exception:  # noqa: BLE001
            self.nvml = None
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()
        t0 = time.perf_counter()
        while not self.samples and time.perf_counter() - t0 < 1.0:
            time.sleep(0.0005)

    def begin(self):
        self.window[0] = time.perf_counter()

    def end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self.stop_evt.set()
        self.thread.join(timeout=5)
        nv = self.nvml
        lo, hi = self.window
        inside = [(m, rs) for t, m, rs in self.samples
                  if (lo is None or t >= lo) and (hi is None or t <= hi)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": ["no samples in the timed region"], "samples": 0}
        reasons = sorted({name for _, rs in inside for name, const in self.REASONS
                          if rs & getattr(nv, const)})
        return {"sm_mhz": statistics.median(m for m, _ in inside),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside)}


class L2Flush:
    """Empties L2 between timed steps: writes one buffer larger than L2, then
    reads another one, so L2 ends up holding only clean lines of the second
    buffer. (A write alone leaves ~126 MB of dirty lines whose write-back the
    next timed kernel would pay for.)"""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def zero_(self):
        self.w.zero_()
        torch.amax(self.r)


def nvtx_push(name):
    try:
        torch.cuda.nvtx.range_push(name)
    except Exception:  # noqa: BLE001 - markers are optional
        pass


def nvtx_pop():
    try:
        torch.cuda.nvtx.range_pop()
    except Exception:  # noqa: BLE001
        pass


def dist_setup(backend="nccl"):
    """Process group for N > 1 ranks (one per GPU). Returns (world, rank, local)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cuda"):
    """The slowest rank's value (the job is as fast as its slowest replica)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(cfg, rank):
    """Inputs of one replica: every rank shares the weights (the model) and gets
    its own batch of tokens; rank 0's batch is the config's own."""
    inp = moe_inputs(cfg)
    if rank > 0:
        gen = torch.Generator().manual_seed(cfg.seed * 1000 + rank)
        inp["x"] = (torch.randn(cfg.t, cfg.d, generator=gen) * inp["x"].float().std()).to(torch.bfloat16)
        inp["logits"] = torch.randn(cfg.t, cfg.n_exp, generator=gen).to(torch.bfloat16)
    return inp


def job_throughput(tokens_per_rank, world, step_s_max):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / step_s_max


# ------------------------------------------------------------ CPU oracle ----
def oracle_weights(cfg, inp, n_experts):
    """Offline oracle quantisation of the first n_experts experts (untimed)."""
    import oracle as O
    wgu_q = np.zeros((cfg.n_exp, 2 * cfg.f, cfg.d), np.int8)
    s_gu = np.zeros((cfg.n_exp, 2 * cfg.f), np.float32)
    wd_q = np.zeros((cfg.n_exp, cfg.d, cfg.f), np.int8)
    s_d = np.zeros((cfg.n_exp, cfg.d), np.float32)
    for e in range(n_experts):
        wgu_q[e], s_gu[e] = O.rotquant(inp["wgu"][e].float().numpy(), cfg.g_gu)
        wd_q[e], s_d[e] = O.rotquant(inp["wd"][e].float().numpy(), cfg.g_d)
    return wgu_q, s_gu, wd_q, s_d


def oracle_cores():
    import threadpoolctl
    threads = max((i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()), default=1)
    return min(threads, len(os.sched_getaffinity(0)))


def oracle_block_time(cfg, inp, weights, n_experts):
    """Seconds for one oracle block call restricted to the first n_experts
    experts' FFN (all routing included), extrapolated per expert to all."""
    import oracle as O
    x = inp["x"].float().numpy()
    logits = inp["logits"].float().numpy()
    t0 = time.perf_counter()
    O.moe_block(x, logits, *weights, cfg.c, cfg.g_gu, cfg.g_d, experts=[])
    t_route = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.moe_block(x, logits, *weights, cfg.c, cfg.g_gu, cfg.g_d, experts=list(range(n_experts)))
    t_sample = time.perf_counter() - t0
    per_expert = max(t_sample - t_route, 0.0) / n_experts
    return t_route + per_expert * cfg.n_exp, t_route + t_sample


def cpu_baseline(cfg, inp, target_s=12.0):
    """The oracle as it stands, full blocks (all experts) repeated until about
    target_s of CPU work; tokens/s over those blocks."""
    import oracle as O
    weights = oracle_weights(cfg, inp, cfg.n_exp)
    x = inp["x"].float().numpy()
    logits = inp["logits"].float().numpy()
    reps, spent = 0, 0.0
    while spent < target_s and reps < 16:
        t0 = time.perf_counter()
        O.moe_block(x, logits, *weights, cfg.c, cfg.g_gu, cfg.g_d)
        spent += time.perf_counter() - t0
        reps += 1
    return {"kind": "oracle", "cores": oracle_cores(), "value": reps * cfg.t / spent, "unit": UNIT,
            "sample": f"{reps} full oracle block(s) on {cfg.name} inputs ({spent:.1f} s of CPU work)"}


def run_reference(args, cfg, world, rank):
    """The oracle timed on the host cores; one step = routing + a quarter of
    the experts' FFN, extrapolated per expert to the whole block."""
    if rank != 0:
        return
    inp = moe_inputs(cfg)
    n_exp = max(1, cfg.n_exp // 4)
    weights = oracle_weights(cfg, inp, n_exp)
    times, spent = [], 0.0
    for _ in range(args.warmup + args.steps):
        block_s, cpu_s = oracle_block_time(cfg, inp, weights, n_exp)
        times.append(block_s)
        spent += cpu_s
    block_s = statistics.mean(times[args.warmup:])
    value = cfg.t / block_s
    info = {"kind": "oracle", "cores": oracle_cores(), "value": value, "unit": UNIT,
            "sample": (f"per step: routing of all {cfg.t} tokens + FFN of experts 0..{n_exp - 1} "
                       f"of {cfg.n_exp} on {cfg.name} inputs, extrapolated per expert to the full "
                       f"block ({spent:.1f} s of CPU work in total)")}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": block_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/int64",
            "data": "synthetic (seeded; stands in for real prompts and trained weights)",
            "config": {"workload": cfg.name, "tokens": cfg.t, "d": cfg.d, "experts": cfg.n_exp,
                       "f": cfg.f, "capacity": cfg.c},
            "cpu_baseline": info,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- GPU path ----
def stage_times(W, ws_views, inp_dev, wq, cfg, t, reps, flush_buf):
    """Device time of every stage, launched through its own C-ABI entry with
    the block's real intermediates, CUDA events on the launching stream."""
    v = ws_views
    gu, dn = wq
    wgu_q, s_gu, wd_q, s_d = gu.data, gu.scale, dn.data, dn.scale
    tiles = W.binding.LAYOUT_TILES
    stream = torch.cuda.current_stream()
    sync = torch.empty(W.binding.lib().convrot_swiglu_rq_sync_bytes(cfg.n_exp, cfg.c),
                       dtype=torch.uint8, device=flush_buf.w.device)
    stages = {
        "router_softmax": lambda: W.binding.lib().convrot_router_softmax(
            W.binding._p(inp_dev["logits"]), t, cfg.n_exp, W.binding._p(v["s_t"]),
            W.binding._stream()),
        "rotquant_x": lambda: W.convrot_rotquant(inp_dev["x"], cfg.g_gu, q=v["x_q"], scale=v["s_x"]),
        "topc": lambda: W.binding.lib().convrot_topc(
            W.binding._p(v["s_t"]), t, cfg.n_exp, cfg.c, W.binding._p(v["idx"]),
            W.binding._p(v["w"]), W.binding._p(v["slot"]), W.binding._stream()),
        "gather": lambda: W.binding.lib().convrot_gather_rows(
            W.binding._p(v["x_q"]), W.binding._p(v["s_x"]), t, W.binding._p(v["idx"]),
            cfg.n_exp * cfg.c, cfg.d, W.binding._p(v["x_g"]), W.binding._p(v["s_g"]),
            W.binding._stream()),
        "gemm_gateup_swiglu": lambda: W.binding.lib().convrot_i8_gemm_swiglu(
            W.binding._p(v["x_g"]), W.binding._p(v["s_g"]), W.binding._p(wgu_q),
            W.binding._p(s_gu), tiles, cfg.n_exp, cfg.c, cfg.f, cfg.d, W.binding._p(v["h"]),
            W.binding._stream()),
        "rotquant_h": lambda: W.convrot_rotquant(v["h"].view(-1, cfg.f), cfg.g_d,
                                                 q=v["h_q"].view(-1, cfg.f), scale=v["s_h"].view(-1)),
        # (the entry clears its 0.1 MB synchronisation scratch first, inside the events)
        "gemm_gateup_swiglu_rq": lambda: W.binding.lib().convrot_i8_gemm_swiglu_rq(
            W.binding._p(v["x_g"]), W.binding._p(v["s_g"]), W.binding._p(wgu_q),
            W.binding._p(s_gu), tiles, cfg.n_exp, cfg.c, cfg.f, cfg.d, cfg.g_d,
            W.binding._p(v["h_q"]), W.binding._p(v["s_h"]), W.binding._p(sync), sync.numel(),
            W.binding._stream()),
        "gemm_down_bf16": lambda: W.binding.lib().convrot_i8_gemm_bf16(
            W.binding._p(v["h_q"]), W.binding._p(v["s_h"]), W.binding._p(wd_q),
            W.binding._p(s_d), tiles, cfg.n_exp, cfg.c, cfg.d, cfg.f,
            W.binding._p(v["z"]), W.binding._stream()),
        "combine": lambda: W.binding.lib().convrot_combine_rows(
            W.binding._p(v["z"]), W.binding._p(v["s_t"]), W.binding._p(v["slot"]), cfg.n_exp, t,
            cfg.c, cfg.d, W.binding._p(inp_dev["y"]), W.binding._stream()),
    }
    # the stages one block call runs
    for name in (("gemm_gateup_swiglu", "rotquant_h") if fused_h(cfg)
                 else ("gemm_gateup_swiglu_rq",)):
        del stages[name]
    out = {}
    for name, fn in stages.items():
        ts = []
        for i in range(reps + 1):
            flush_buf.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rc = fn()
            b.record(stream)
            if isinstance(rc, int) and rc != 0:
                raise RuntimeError(f"stage {name} failed: {rc}")
            torch.cuda.synchronize()
            if i > 0:
                ts.append(a.elapsed_time(b) * 1e-3)
        out[name] = statistics.median(ts)
    return out


def timed(fn, steps, flush_buf, stream):
    """Device seconds of each of `steps` calls of fn (L2 flushed before each,
    outside the events; CUDA events on the launching stream)."""
    out = []
    for _ in range(steps):
        flush_buf.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        out.append(a.elapsed_time(b) * 1e-3)
    return out


def block_workload(W, cfg, wq, ws, flush_buf, steps, warmup, dev, stream):
    """The block at cfg's T on cfg's own tokens and logits, with the weights
    wq (the same model at every T). Returns its measurements."""
    inp = moe_inputs(cfg, weights=False)
    x, logits = inp["x"].to(dev), inp["logits"].to(dev)
    y = torch.empty((cfg.t, cfg.d), dtype=torch.bfloat16, device=dev)
    gu, dn = wq

    def step():
        W.moe_expert_choice_forward(x, logits, gu, dn, cfg.c, cfg.g_gu, cfg.g_d, y=y, workspace=ws)

    timed(step, warmup, flush_buf, stream)
    st = statistics.mean(timed(step, steps, flush_buf, stream))
    work = algorithmic_work(cfg, cfg.t)
    return {"tokens": cfg.t, "capacity": cfg.c, "ms_per_step": st * 1e3, "tokens_per_s": cfg.t / st,
            "block": roofline_of(work["ops"], work["block_bytes"], st, load_peaks())}


def lowbit_work(cfg, t, bits):
    """Ops and compulsory bytes of the block with b-bit expert weights: the
    packed codes (bits/8 bytes per weight), one E4M3 byte per 16 weights and
    the FP32 row scales once, X and logits in, Y out; and of its two GEMMs
    (weights + scales)."""
    e, c, d, f = cfg.n_exp, cfg.c, cfg.d, cfg.f

    def wbytes(n_w, rows):
        return n_w * bits // 8 + n_w // 16 + rows * 4

    gu = wbytes(e * 2 * f * d, e * 2 * f)
    dn = wbytes(e * d * f, e * d)
    return {"ops": 2 * e * c * (d * 2 * f + f * d),
            "block_bytes": gu + dn + t * d * 2 + t * e * 2 + t * d * 2,
            "gateup_alg": {"ops": 2 * e * c * d * 2 * f, "bytes": gu},
            "down_alg": {"ops": 2 * e * c * f * d, "bytes": dn}}


def roofline_f16(ops, nbytes, seconds, peaks):
    """Both fractions for the low-bit path, whose contraction runs on the
    kind::f16 tensor cores: the tensor peak is the measured bf16 burst (f16
    and bf16 have the same dense rate)."""
    tc = peaks["bf16_tflops"]
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = ops / (tc * 1e12)
    gbs = nbytes / seconds / 1e9
    tops = ops / seconds / 1e12
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor",
            "ideal_us": max(t_hbm, t_tc) * 1e6, "roofline_frac": max(t_hbm, t_tc) / seconds,
            "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
            "tflops": tops, "tensor_frac": tops / tc}


def lowbit_workloads(W, wgu, wd, g_gu, g_d, flush_buf, steps, dev, stream,
                     names=("moe_T512", "moe_T2048", "moe_T8192")):
    """The MoE block with W4A8 and W6A8 expert weights (the same bf16 model
    quantised to the b-bit formats) at several T, and its two GEMMs alone on
    the call's own intermediates."""
    peaks = load_peaks()
    out = {}
    for bits in (4, 6):
        gu, dn = W.quantize_moe_weights_lowbit(wgu, wd, bits, g_gu, g_d)
        for name in names:
            cfg = MOE_CONFIGS[name]
            inp = moe_inputs(cfg, weights=False)
            x, logits = inp["x"].to(dev), inp["logits"].to(dev)
            y = torch.empty((cfg.t, cfg.d), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(W.moe_workspace_size(cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c),
                             dtype=torch.uint8, device=dev)

            def step():
                W.moe_expert_choice_forward_lowbit(x, logits, gu, dn, cfg.c, g_gu, g_d, y=y,
                                                   workspace=ws)

            timed(step, 3, flush_buf, stream)
            st = statistics.mean(timed(step, steps, flush_buf, stream))
            v = W.moe_stage_views(ws, cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c)
            g1 = lambda: W.convrot_lowbit_gemm(v["x_g"], v["s_g"], gu, W.CONVROT_LOWBIT_SWIGLU,  # noqa: E731
                                               out=v["h"])
            g2 = lambda: W.convrot_lowbit_gemm(v["h_q"], v["s_h"], dn, W.CONVROT_LOWBIT_BF16,  # noqa: E731
                                               out=v["z"])
            timed(g1, 3, flush_buf, stream)
            t1 = statistics.median(timed(g1, steps, flush_buf, stream))
            timed(g2, 3, flush_buf, stream)
            t2 = statistics.median(timed(g2, steps, flush_buf, stream))
            work = lowbit_work(cfg, cfg.t, bits)
            out[f"w{bits}a8_{name}"] = {
                "bits": bits, "tokens": cfg.t, "capacity": cfg.c,
                "ms_per_step": st * 1e3, "tokens_per_s": cfg.t / st,
                "block": roofline_f16(work["ops"], work["block_bytes"], st, peaks),
                "gemm_gateup_swiglu_us": t1 * 1e6,
                "gemm_gateup_swiglu": roofline_f16(work["gateup_alg"]["ops"],
                                                   work["gateup_alg"]["bytes"], t1, peaks),
                "gemm_down_bf16_us": t2 * 1e6,
                "gemm_down_bf16": roofline_f16(work["down_alg"]["ops"], work["down_alg"]["bytes"],
                                               t2, peaks)}
            del ws
        del gu, dn
    return out


def linear_workloads(W, flush_buf, reps, dev, stream, configs=None):
    """The single W8A8 ConvRot linears through w8a8_convrot_linear (rotation +
    GEMM), and the GEMM alone on the same codes (convrot_i8_gemm_bf16)."""
    peaks = load_peaks()
    out = {}
    for name, cfg in (LINEAR_CONFIGS if configs is None else configs).items():
        x, w = linear_inputs(cfg)
        x, w = x.to(dev), w.to(dev)
        w_q, s_w = W.convrot_quantize_weights(w, cfg.group)
        ws = torch.empty(max(W.convrot_linear_workspace_size(cfg.m, cfg.k), 16), dtype=torch.uint8,
                         device=dev)
        y = torch.empty((cfg.m, cfg.n), dtype=torch.bfloat16, device=dev)
        lin = lambda: W.w8a8_convrot_linear(x, w_q, s_w, cfg.group, y=y, workspace=ws)  # noqa: E731
        timed(lin, 3, flush_buf, stream)
        t_lin = statistics.median(timed(lin, reps, flush_buf, stream))
        x_q = ws[:cfg.m * cfg.k].view(torch.int8).view(cfg.m, cfg.k)
        off = (cfg.m * cfg.k + 255) // 256 * 256
        s_x = ws[off:off + 4 * cfg.m].view(torch.float32)
        gemm = lambda: W.convrot_i8_gemm_bf16(x_q, s_x, w_q, s_w)  # noqa: E731
        timed(gemm, 3, flush_buf, stream)
        t_gemm = statistics.median(timed(gemm, reps, flush_buf, stream))
        ops = 2 * cfg.m * cfg.n * cfg.k
        # the linear's algorithmic bytes: X in (bf16), codes and scales of W, Y out (bf16)
        nbytes = cfg.m * cfg.k * 2 + cfg.n * cfg.k + cfg.n * 4 + cfg.m * cfg.n * 2
        gemm_bytes = cfg.m * cfg.k + cfg.m * 4 + cfg.n * cfg.k + cfg.n * 4 + cfg.m * cfg.n * 2
        out[name] = {"m": cfg.m, "n": cfg.n, "k": cfg.k, "group": cfg.group,
                     "linear_us": t_lin * 1e6, "linear": roofline_of(ops, nbytes, t_lin, peaks),
                     "gemm_us": t_gemm * 1e6, "gemm": roofline_of(ops, gemm_bytes, t_gemm, peaks)}
    return out


def int8_peak_probe(W, flush_buf, dev, stream, n=8192, reps=10):
    """Dense INT8 tensor throughput this library's own GEMM reaches: one
    n x n x n product of random codes with the bf16 epilogue (the output is
    1/n of the work), best of `reps`. A lower bound on the hardware's peak."""
    gen = torch.Generator(device=dev).manual_seed(0)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=gen)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=gen)
    s_a = torch.full((n,), 1e-3, device=dev)
    s_b = torch.full((n,), 1e-3, device=dev)
    fn = lambda: W.convrot_i8_gemm_bf16(a, s_a, b, s_b)  # noqa: E731
    timed(fn, 3, flush_buf, stream)
    best = min(timed(fn, reps, flush_buf, stream))
    tops = 2.0 * n ** 3 / best / 1e12
    peaks = load_peaks()
    return {"shape": f"{n}x{n}x{n}", "us": best * 1e6, "tops": tops,
            "of_2x_bf16_measured": tops / (2.0 * peaks["bf16_tflops"]),
            "of_datasheet": tops / INT8_DATASHEET_TOPS}


def run_ours(args, cfg, world, rank, local, extras=True):
    import w8a8_rotated_int8_b200 as W
    W.load_library()
    W.convrot_device_check()
    dev = torch.device("cuda", local)
    t = cfg.t
    inp = rank_inputs(cfg, rank)
    gu, dn = W.quantize_moe_weights(inp["wgu"].to(dev), inp["wd"].to(dev), cfg.g_gu, cfg.g_d)
    wq = (gu, dn)
    x = inp["x"].to(dev)
    logits = inp["logits"].to(dev)
    y = torch.empty((t, cfg.d), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(W.moe_workspace_size(t, cfg.d, cfg.f, cfg.n_exp, cfg.c), dtype=torch.uint8,
                     device=dev)
    flush_buf = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step(xx, ll, yy):
        W.moe_expert_choice_forward(xx, ll, gu, dn, cfg.c, cfg.g_gu, cfg.g_d, y=yy, workspace=ws)

    for _ in range(args.warmup):
        flush_buf.zero_()
        step(x, logits, y)
    torch.cuda.synchronize()
    if W.convrot_check_device_error() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")
    # the timed steps replay one call captured in a CUDA graph (what a serving
    # loop does; the host's launch work then stays out of the device timing)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(x, logits, y)
    torch.cuda.synchronize()
    for _ in range(2):
        flush_buf.zero_()
        graph.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev)
    clocks.start()  # sampling from here on; only the timed window below is reported
    barrier(world)
    torch.cuda.synchronize()
    clocks.begin()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    wall0 = time.perf_counter()
    nvtx_push("timed_steps")  # lets an ncu run select exactly these launches (--nvtx)
    for i in range(args.steps):
        flush_buf.zero_()  # L2 flush (write, then read), outside the timed events
        starts[i].record(stream)
        graph.replay()
        ends[i].record(stream)
    nvtx_pop()
    torch.cuda.synchronize()
    clocks.end()
    barrier(world)
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    del graph
    step_s = [s.elapsed_time(e) * 1e-3 for s, e in zip(starts, ends)]
    mean_step = max_over_ranks(statistics.mean(step_s), world)

    # end to end through the C ABI with host buffers: pinned inputs in, result out
    x_h = inp["x"].pin_memory()
    l_h = inp["logits"].pin_memory()
    y_h = torch.empty((t, cfg.d), dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        x.copy_(x_h, non_blocking=True)
        logits.copy_(l_h, non_blocking=True)
        step(x, logits, y)
        y_h.copy_(y, non_blocking=True)

    timed(e2e_step, 2, flush_buf, stream)
    e2e_serial_s = max_over_ranks(
        statistics.mean(timed(e2e_step, min(args.steps, 20), flush_buf, stream)), world)

    # the same calls as a serving loop runs them: step i+1's inputs copied in
    # and step i-1's result copied out while step i runs (two device buffer
    # sets; copies in, the call, copies out on three streams); the L2 flush
    # before every call is inside the timing here
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [(torch.empty_like(x), torch.empty_like(logits), torch.empty_like(y)) for _ in range(2)]

    def e2e_pipelined(n):
        torch.cuda.synchronize()
        t_a = torch.cuda.Event(enable_timing=True)
        t_b = torch.cuda.Event(enable_timing=True)
        t_a.record(stream)
        cin.wait_stream(stream)
        cout.wait_stream(stream)
        done, out = [], []
        for i in range(n):
            xb, lb, yb = sets[i % 2]
            if i >= 2:
                cin.wait_event(done[i - 2])     # the set's inputs consumed
            with torch.cuda.stream(cin):
                xb.copy_(x_h, non_blocking=True)
                lb.copy_(l_h, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(cin)
            stream.wait_event(ready)
            if i >= 2:
                stream.wait_event(out[i - 2])   # the set's result copied out
            flush_buf.zero_()
            step(xb, lb, yb)
            ev = torch.cuda.Event()
            ev.record(stream)
            done.append(ev)
            cout.wait_event(ev)
            with torch.cuda.stream(cout):
                y_h.copy_(yb, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(cout)
                out.append(ev)
        stream.wait_event(out[-1])
        t_b.record(stream)
        t_b.synchronize()
        return t_a.elapsed_time(t_b) * 1e-3 / n

    e2e_pipelined(3)
    e2e_step_s = max_over_ranks(e2e_pipelined(args.steps), world)

    # per-stage device times (dominant kernel for the roofline)
    views = W.moe_stage_views(ws, t, cfg.d, cfg.f, cfg.n_exp, cfg.c)
    st = stage_times(W, views, {"x": x, "logits": logits, "y": y}, wq, cfg, t, 5, flush_buf)
    flags = W.convrot_check_device_error()
    if flags != 0:
        raise RuntimeError(f"device error flags {flags:#x}")

    # the other workloads of the same model, on rank 0 only (N = 1 lines)
    workloads = {}
    if extras and world == 1:
        big = torch.empty(W.moe_workspace_size(8192, cfg.d, cfg.f, cfg.n_exp, 256),
                          dtype=torch.uint8, device=dev) if t < 8192 else ws
        for name in ("moe_T512", "moe_T1024", "moe_T2048", "moe_T4096", "moe_T8192"):
            other = MOE_CONFIGS[name]
            if other.t == t:
                continue
            workloads[name] = block_workload(W, other, wq, big, flush_buf, 20, 3, dev, stream)
        del big
        workloads["linears"] = linear_workloads(W, flush_buf, 10, dev, stream)
        dit = linear_workloads(W, flush_buf, 5, dev, stream, DIT_LINEARS)
        tot_us = sum(v["linear_us"] for v in dit.values())
        tot_ops = sum(2 * v["m"] * v["n"] * v["k"] for v in dit.values())
        dit["block"] = {"linears": len(DIT_LINEARS), "linear_us_sum": tot_us,
                        "tops": tot_ops / tot_us / 1e6,
                        "tensor_frac": tot_ops / tot_us / 1e6 / (2.0 * load_peaks()["bf16_tflops"])}
        workloads["dense_dit_block"] = dit
        workloads["int8_gemm_probe"] = int8_peak_probe(W, flush_buf, dev, stream)
        workloads["lowbit"] = lowbit_workloads(W, inp["wgu"].to(dev), inp["wd"].to(dev), cfg.g_gu,
                                               cfg.g_d, flush_buf, 10, dev, stream)
        flags = W.convrot_check_device_error()
        if flags != 0:
            raise RuntimeError(f"device error flags {flags:#x}")

    if rank != 0:
        return
    peaks = load_peaks()
    work = algorithmic_work(cfg, t)
    gateup_stage = "gemm_gateup_swiglu_rq" if fused_h(cfg) else "gemm_gateup_swiglu"
    dom = max((gateup_stage, "gemm_down_bf16"), key=lambda k: st[k])
    dk = work["down_alg"] if dom == "gemm_down_bf16" else work["gateup_alg"]
    kr = roofline_of(dk["ops"], dk["bytes"], st[dom], peaks)
    int8_peak = 2.0 * peaks["bf16_tflops"]
    if kr["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": kr["hbm_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kr["hbm_frac"]}
    else:
        roof = {"bound": "tensor", "achieved": kr["tops"], "peak": int8_peak, "unit": "TOPS",
                "frac": kr["tensor_frac"]}
    traffic, traffic_note = profile_traffic(dom, cfg.name)
    if args.traffic_bytes is not None:
        traffic, traffic_note = args.traffic_bytes, "given on the command line"
    roof.update({
        "scope": f"dominant kernel ({dom}); the whole block is under block_roofline",
        "traffic": traffic, "traffic_source": traffic_note,
        "hbm_frac": kr["hbm_frac"], "tensor_frac": kr["tensor_frac"],
        "tensor_frac_datasheet": kr["tensor_frac_datasheet"],
        "kernel_us": st[dom] * 1e6, "algorithmic_bytes": dk["bytes"], "algorithmic_ops": dk["ops"],
        "bytes_rule": "expert weights once + their scales (gathered and intermediate copies excluded)",
        "peak_source": (f"{peaks['source']}: HBM copy {peaks['hbm_gbs']} GB/s; INT8 "
                        f"{int8_peak:.0f} TOPS = 2 x measured bf16 burst"),
    })
    block = roofline_of(work["ops"], work["block_bytes"], mean_step, peaks)

    value = job_throughput(t, world, mean_step)
    # softmax, rotation, top-C, [gather, GEMM, (h rotation,) GEMM], combine
    launches_per_step = (7 if fused_h(cfg) else 8) if cfg.c > 0 else 4
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 (int32 acc, fp32 epilogue)",
        "data": "synthetic (seeded; stands in for real prompts and trained weights)",
        "config": {"workload": cfg.name, "tokens_per_gpu": t, "d": cfg.d, "experts": cfg.n_exp,
                   "f": cfg.f, "capacity": cfg.c, "g_gu": cfg.g_gu, "g_d": cfg.g_d,
                   "parallelism": f"replicas x{world} (independent batches)",
                   "launch": "timed steps replay one captured CUDA graph of the call; e2e calls it eagerly",
                   "l2": "flushed before every step (256 MiB write + 256 MiB read, outside the timed events)"},
        "roofline_block_frac": block["roofline_frac"],
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": job_throughput(t, world, e2e_step_s), "unit": UNIT,
                "h2d_bytes_per_step": int(x_h.numel() * 2 + l_h.numel() * 2),
                "d2h_bytes_per_step": int(y_h.numel() * 2),
                "overlap": "copies of neighbouring steps overlap the call (two buffer sets, "
                           "three streams); L2 flushed before every call inside the timing",
                "serial_value": job_throughput(t, world, e2e_serial_s)},
        "roofline": roof,
        "block_roofline": {**block, "algorithmic_bytes": work["block_bytes"], "ops": work["ops"]},
        "stage_us": {k: v * 1e6 for k, v in st.items()},
        "clocks": clk,
        "wall_s": wall,
    }
    if workloads:
        line["workloads"] = workloads
    if args.cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(cfg, inp)
    print(json.dumps(line), flush=True)


def run_ablation(args, cfg):
    """Rotation-off ablation on the block (g_gu = g_d = 1: per-token and
    per-channel INT8 with no Hadamard, the same kernels) against ConvRot
    (the config's groups): the relative error of each block output against an
    unquantised fp32 evaluation of the same routed experts (bf16 inputs and
    weights, torch matmuls), on a sample of tokens. Prints one JSON line."""
    import w8a8_rotated_int8_b200 as W
    W.load_library()
    dev = torch.device("cuda", 0)
    inp = moe_inputs(cfg)
    x = inp["x"].to(dev)
    logits = inp["logits"].to(dev)
    wgu = inp["wgu"].to(dev)
    wd = inp["wd"].to(dev)
    ws = torch.empty(W.moe_workspace_size(cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c), dtype=torch.uint8,
                     device=dev)
    gen = torch.Generator().manual_seed(7)
    sample = torch.randperm(cfg.t, generator=gen)[:256].sort().values.to(dev)
    result = {}
    ref = None
    for name, g_gu, g_d in (("convrot", cfg.g_gu, cfg.g_d), ("rotation_off", 1, 1)):
        gu, dn = W.quantize_moe_weights(wgu, wd, g_gu, g_d)
        y = W.moe_expert_choice_forward(x, logits, gu, dn, cfg.c, g_gu, g_d, workspace=ws)
        torch.cuda.synchronize()
        v = W.moe_stage_views(ws, cfg.t, cfg.d, cfg.f, cfg.n_exp, cfg.c)
        if ref is None:  # routing does not depend on the groups
            ref = torch.zeros(cfg.t, cfg.d, dtype=torch.float32, device=dev)
            idx = v["idx"].long()
            s_t = v["s_t"]
            keep = torch.zeros(cfg.t, dtype=torch.bool, device=dev)
            keep[sample] = True
            for e in range(cfg.n_exp):
                rows = idx[e][keep[idx[e]]]
                if rows.numel() == 0:
                    continue
                xe = x[rows].float()
                gu_out = xe @ wgu[e].float().t()
                h = torch.nn.functional.silu(gu_out[:, :cfg.f]) * gu_out[:, cfg.f:]
                ref[rows] += s_t[e, rows][:, None] * (h @ wd[e].float().t())
        ys, rs = y[sample].float(), ref[sample]
        result[name] = {
            "g_gu": g_gu, "g_d": g_d,
            "max_rel": float((ys - rs).abs().max() / rs.abs().max()),
            "rel_fro": float(torch.linalg.norm(ys - rs) / torch.linalg.norm(rs)),
        }
        del gu, dn
    line = {"metric": "W8A8 MoE block relative error vs an unquantised fp32 evaluation "
                      "(rotation-off ablation)",
            "config": {"workload": cfg.name, "tokens_sampled": int(sample.numel())},
            "data": "synthetic (seeded; 1% of the activation channels x20 as outliers)",
            **result}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="moe_T8192", choices=sorted(MOE_CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="only the configured block (no other T, linears or INT8 probe)")
    ap.add_argument("--only-linears", action="store_true",
                    help="only the single W8A8 ConvRot linears and the dense-DiT block's linears "
                         "(one JSON line; used to profile the linear GEMMs)")
    ap.add_argument("--only-lowbit", action="store_true",
                    help="only the W4A8 / W6A8 blocks and their GEMMs (one JSON line)")
    ap.add_argument("--ablation", action="store_true",
                    help="rotation-off ablation: block error with and without ConvRot")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per token count T in 512..8192 (C = 2T/64), no CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = MOE_CONFIGS[args.config]
    if args.ablation:
        run_ablation(args, cfg)
        return
    if args.only_linears:
        import w8a8_rotated_int8_b200 as W
        W.load_library()
        dev = torch.device("cuda", 0)
        flush_buf = L2Flush(dev)
        stream = torch.cuda.current_stream()
        line = {"metric": "W8A8 ConvRot linears", "data": "synthetic (seeded)",
                "linears": linear_workloads(W, flush_buf, args.steps, dev, stream),
                "dense_dit_block": linear_workloads(W, flush_buf, args.steps, dev, stream,
                                                    DIT_LINEARS)}
        print(json.dumps(line), flush=True)
        return
    if args.only_lowbit:
        import w8a8_rotated_int8_b200 as W
        W.load_library()
        dev = torch.device("cuda", 0)
        inp = moe_inputs(cfg)
        line = {"metric": "W4A8 / W6A8 ConvRot MoE block", "data": "synthetic (seeded)",
                "lowbit": lowbit_workloads(W, inp["wgu"].to(dev), inp["wd"].to(dev), cfg.g_gu,
                                           cfg.g_d, L2Flush(dev), args.steps, dev,
                                           torch.cuda.current_stream())}
        if W.convrot_check_device_error() != 0:
            raise RuntimeError("device error flags set")
        print(json.dumps(line), flush=True)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, cfg, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        if args.sweep:
            args.cpu_baseline = False
            for name in ("moe_T512", "moe_T1024", "moe_T2048", "moe_T4096", "moe_T8192"):
                run_ours(args, MOE_CONFIGS[name], world, rank, local, extras=False)
        else:
            run_ours(args, cfg, world, rank, local, extras=args.extras)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
