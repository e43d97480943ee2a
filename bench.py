#!/usr/bin/env python
"""Benchmark of the block-scaled GEMM path on B200.

One step = the whole hot path on one batch of synthetic input: pack the UE8M0 scale
factors of A (1x128) and B (128x128) into int16 MN-major words on the GPU, then the FP8
E4M3 block-scaled GEMM D = A * B^T at M=4096 N=7168 K=16384 (fp32 accumulate, bf16 out).
The L2 is flushed (1 GiB write) before every timed step; the flush is outside the events.

The same line also reports, each measured the same way (W warm-up, flushed L2, CUDA
events on the launching stream): BF16 dense at the same shape, FP4 E2M1 at the same
shape, the M-grouped FP8 MoE workload (32 experts, 32768 rows, N=4096, K=7168), the FP8
M sweep {128, 1024, 4096} at N=K=7168, the masked grouped (decode) layout (32 experts x 256
rows, N=4096, K=7168), the scale transform alone (GB/s), and the FP8
quantiser that produces the GEMM's operands (fp32 A in 1x128 blocks, bf16 B in 128x128
blocks, GB/s).

FLOP convention 2*M*N*K per GEMM (the pages' own timings reproduce their TFLOPS with it).

--impl reference times the CPU oracle (the plain fp64 definition) on bounded row samples
of the same FP8 workload; it is a deliberately slow reference, not a target.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import inputs  # noqa: E402

METRIC = "GEMM TFLOPS (FP8 block-scaled, BF16) at 4096×7168×16384; % of B200 peak"
M, N, K = 4096, 7168, 16384
PAGES_FP8_TFLOPS = 861.0   # pages' FP8xFP8 figure at this shape (Ascend 950DT): context only
PAGES_BF16_TFLOPS = 431.0
NOMINAL_RATIO = {"bf16": 1.0, "fp8": 2.0, "fp4": 4.0}  # dense tensor peak relative to bf16
# dense tcgen05 MMA throughput per SM per clock, and the spec sheet's dense peaks per GPU
PER_SM_FLOPS_PER_CLK = {"bf16": 8192, "fp8": 16384, "fp4": 32768}
SPEC_PEAK_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0, "fp4": 9000.0}
SECONDARY_REPS = 50  # samples per secondary workload (after the warm-up)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = "block_scaled_precision_sm_b200/csrc/"
# the sources each profiled kernel depends on (device code and the host code that launches it)
KERNEL_SOURCES = {
    "gemm": [_CSRC + f for f in ("gemm.cuh", "ptx.cuh", "sf_layout.cuh", "api.cu")],
    "sf_transform": [_CSRC + f for f in ("sf_transform.cuh", "ptx.cuh", "api.cu", "sf_batch.cu")],
    "quantize": [_CSRC + f for f in ("quantize.cuh", "quantize.cu")],
}


def workload_config(world: int, shard: str = "none", gather: bool = False) -> dict:
    """The headline workload, as both arms report it."""
    if shard == "n":
        par = (f"n-sharded x{world}: one 4096x7168x16384 problem, rank r computes D[:, n0:n1] from all of A "
               f"and rows [n0, n1) of B (128-aligned shards of N)" +
               ("; the step ends with an all-gather of D over the process group" if gather and world > 1
                else "; no collective in the step"))
    else:
        par = f"one independent problem per GPU x{world}"
    return {"workload": "fp8_block_scaled_gemm_nt 4096x7168x16384 (sf transform + gemm)", "M": M, "N": N,
            "K": K, "sfa": "1x128 ue8m0", "sfb": "128x128 ue8m0",
            "l2": "flushed by a 1 GiB write before every step, outside the events",
            "parallelism": par}


def gemm_flops(m: int, n: int, k: int) -> float:
    return 2.0 * m * n * k


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--only-headline", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--shard", choices=["none", "n"], default="none",
                    help="none: one independent problem per GPU (weak scaling); n: one problem split along N "
                         "over the ranks (strong scaling)")
    ap.add_argument("--gather", action="store_true", help="with --shard n: all-gather D inside every step")
    ap.add_argument("--profile", choices=["fp8", "fp8_m128", "fp8_m1024", "fp8_m4096", "bf16", "fp4", "grouped", "masked",
                                          "sf_transform", "sf_transform_64x", "sf_transform_fp4", "quantize_act",
                                          "quantize_wgt"],
                    help="launch only this kernel (warm-up + steps launches, no timing) for an ncu capture")
    return ap.parse_args()


def rank_env():
    """(rank, world size, local rank) of this process, as torchrun sets them."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """The source with comments, trailing blanks and empty lines removed: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line)


def sources_digest(kind: str = "gemm") -> str:
    """Digest of the code (not the comments) of the sources a profiled kernel depends on."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on these sources."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    s = re.search(r"sources_digest:\s*([0-9a-f]+)", txt)
    kind = "quantize" if name.startswith("quantize") else "sf_transform" if name.startswith("sf_transform") else "gemm"
    if not t or not s or s.group(1) != sources_digest(kind):
        return None
    return float(t.group(1))


# ---------------------------------------------------------------- clocks sampler

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled every `period_s` by a
    thread for the whole run (NVML, the library nvidia-smi reads), so that even a timed region
    of a few milliseconds holds several samples.  window(t0, t1) summarises the samples taken
    between two perf_counter() stamps."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, cuda_index: int, period_s: float = 0.001):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []  # (perf_counter, sm MHz, power W, reason bits)
        self.error = None
        self._stop = None
        self._thread = None
        self.max_mhz = None

    def _handle(self, nv):
        import torch

        props = torch.cuda.get_device_properties(self.cuda_index)
        try:
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:  # noqa: BLE001
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)

    def start(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception as e:  # noqa: BLE001
            self.error = f"nvml unavailable: {e}"
            return
        self._stop = threading.Event()
        first = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    t = time.perf_counter()
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    self.samples.append((t, mhz, watts, bits))
                except Exception as e:  # noqa: BLE001
                    self.error = str(e)
                first.set()
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        first.wait(5.0)  # the first sample exists before any timed region starts

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5.0)

    def window(self, t0: float | None = None, t1: float | None = None) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.error or "no samples"],
                    "samples": 0}
        import pynvml as nv

        sel = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not sel:  # a window shorter than one period: the samples bracketing it
            before = [x for x in self.samples if x[0] < t0]
            after = [x for x in self.samples if x[0] > t1]
            sel = before[-1:] + after[:1]
        mhz = [x[1] for x in sel]
        reasons = sorted({name for name, attr in self.REASONS for x in sel if x[3] & getattr(nv, attr)})
        return {"sm_mhz": statistics.median(mhz), "sm_mhz_min": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sel), "power_w_max": round(max(x[2] for x in sel), 1),
                "source": "nvml, 1 ms period"}


def spread(ms: np.ndarray) -> dict:
    """Median, p10 and p90 of per-step times (ms) beside their mean."""
    return {"median_ms": round(float(np.median(ms)), 5), "p10_ms": round(float(np.percentile(ms, 10)), 5),
            "p90_ms": round(float(np.percentile(ms, 90)), 5), "mean_ms": round(float(np.mean(ms)), 5),
            "samples": int(len(ms))}


# ---------------------------------------------------------------- our arm

class Timer:
    """Per-step CUDA events on the launching stream, L2 flushed before each step."""

    def __init__(self, torch, flush_bytes=1 << 30):
        self.torch = torch
        self.flush = torch.empty(flush_bytes, dtype=torch.uint8, device="cuda")

    def run(self, fn, warmup: int, steps: int, marks: int = 1):
        torch = self.torch
        for _ in range(warmup):
            self.flush.zero_()
            fn(None)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(marks + 1)] for _ in range(steps)]
        for i in range(steps):
            self.flush.zero_()
            fn(evs[i])
        torch.cuda.synchronize()
        spans = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(marks)] for i in range(steps)])
        return spans  # ms, [steps, marks]


def fp8_device_problem(torch, m, n, k, seed):
    p = inputs.dense_fp8_problem(m, n, k, seed=seed)
    dev = {key: torch.from_numpy(p[key]).cuda() for key in ("A", "sfa", "B", "sfb")}
    return p, dev


def peak_fractions(achieved_tflops: float, dtype: str, sms: int, clocks: dict) -> dict:
    """The achieved rate against the dense tensor peak two other ways: the spec sheet's figure
    and the clock-derived peak (SMs x dense MMA flops per SM per clock x SM clock), at the
    median SM clock sampled during the timing and at the maximum clock."""
    per_clk = PER_SM_FLOPS_PER_CLK[dtype] * sms
    out = {"spec_peak_tflops": SPEC_PEAK_TFLOPS[dtype],
           "frac_of_spec": round(achieved_tflops / SPEC_PEAK_TFLOPS[dtype], 4)}
    for key, mhz in (("at_sampled_clock", clocks.get("sm_mhz")), ("at_max_clock", clocks.get("sm_max_mhz"))):
        if mhz:
            peak = per_clk * mhz * 1e6 / 1e12
            out[f"clock_peak_tflops_{key}"] = round(peak, 1)
            out[f"frac_of_clock_peak_{key}"] = round(achieved_tflops / peak, 4)
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    from block_scaled_precision_sm_b200 import ops

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks, peak_kind = load_peaks()
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    sampler = ClockSampler(local)
    sampler.start()

    timer = Timer(torch)
    kb = K // 128
    sharded = args.shard == "n"
    gather = sharded and args.gather and world > 1
    if sharded:
        # one problem for the whole job: every rank draws the same operands and keeps its rows of B
        from block_scaled_precision_sm_b200 import shard

        p = inputs.dense_fp8_problem(M, N, K, seed=100)
        bounds = shard.n_shard_bounds(N, world)
        n0, n1 = bounds[rank]
        p["B"], p["sfb"] = p["B"][n0:n1], p["sfb"][n0 // 128:-(-n1 // 128)]
        dev = {key: torch.from_numpy(np.ascontiguousarray(p[key])).cuda() for key in ("A", "sfa", "B", "sfb")}
    else:
        # independent problem per rank (weak scaling): the seed differs by rank
        n0, n1 = 0, N
        p, dev = fp8_device_problem(torch, M, N, K, seed=100 + 7 * rank)
    n_local = n1 - n0
    sfa_w = torch.empty(((kb + 1) // 2, ops.sf_ld(M)), dtype=torch.int16, device="cuda")
    sfb_w = torch.empty(((kb + 1) // 2, ops.sf_ld(-(-n_local // 128))), dtype=torch.int16, device="cuda")
    D = torch.empty((M, n_local), dtype=torch.bfloat16, device="cuda")

    def step(ev):
        if ev is not None:
            ev[0].record()
        ops.transform_sf_ue8m0_pair(dev["sfa"], dev["sfb"], out_a=sfa_w, out_b=sfb_w)  # both scale tensors
        if ev is not None:
            ev[1].record()
        ops.gemm_fp8_nt(dev["A"], sfa_w, dev["B"], sfb_w, D, sfb_gran_n=128)
        if ev is not None:
            ev[2].record()
        if gather:
            shard.all_gather_columns(D, bounds)
        if ev is not None:
            ev[3].record()

    # warm-up + timed region bracketed by barrier and synchronize on both sides
    for _ in range(args.warmup):
        timer.flush.zero_()
        step(None)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    launches0 = ops.kernel_launches()
    wall0 = time.perf_counter()
    spans = timer.run(step, 0, args.steps, marks=3)
    wall1 = time.perf_counter()
    launches = ops.kernel_launches() - launches0
    torch.cuda.synchronize()
    barrier(world)
    status = ops.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    clocks = sampler.window(wall0, wall1)

    step_ms = max_over_ranks(float(spans.sum(axis=1).mean()), world, "cuda")
    gemm_ms = max_over_ranks(float(spans[:, 1].mean()), world, "cuda")
    flops = gemm_flops(M, n_local, K)  # this rank's launch
    job_flops = gemm_flops(M, N, K) * (1 if sharded else world)
    value = job_flops / (step_ms * 1e-3) / 1e12
    fp8_peak = peaks["bf16_tflops"] * NOMINAL_RATIO["fp8"]
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    traffic = profiled_traffic("gemm_fp8_4096x7168x16384.md")
    plan = ops.gemm_plan("fp8", M, N, K)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": round(value / world / PAGES_FP8_TFLOPS, 3),
        "vs_baseline_note": "per-GPU value / the pages' 861 TFLOPS FP8xFP8 at this shape on an Ascend 950DT "
                            "(another machine: context, not the target)",
        "dtype": "e4m3 x ue8m0 scales, fp32 accumulate, bf16 out", "data": "synthetic",
        "config": workload_config(world, args.shard, args.gather),
        "step_time": spread(spans.sum(axis=1)),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 burst x 2 (nominal fp8/bf16 ratio)",
                     "frac_of_sustained": round(achieved / (peaks.get("bf16_tflops_sustained", 1400.0) * 2), 4),
                     **peak_fractions(achieved, "fp8", sms, clocks),
                     "kernel": "gemm_kernel<FP8, {tile_m}x{tile_n} pair tiles>".format(**plan),
                     "plan": plan, "gemm_call_ms": round(gemm_ms, 5),
                     "gemm_call_time": spread(spans[:, 1]),
                     "timed_span": "CUDA events around the gemm_fp8_nt call: its scale-chunk prepass kernel "
                                   "and the GEMM kernel (launched to overlap the prepass)"},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "wall_s_timed_region": round(wall1 - wall0, 4),
    }

    # end to end through the public API: pinned host inputs -> GPU -> host result, every step
    pin = {key: torch.from_numpy(np.ascontiguousarray(p[key])).pin_memory() for key in ("A", "sfa", "B", "sfb")}
    D_host = torch.empty((M, n_local), dtype=torch.bfloat16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = D_host.numel() * D_host.element_size()

    def e2e_step(ev):
        if ev is not None:
            ev[0].record()
        for key in pin:
            dev[key].copy_(pin[key], non_blocking=True)
        ops.gemm_fp8_nt(dev["A"], dev["sfa"], dev["B"], dev["sfb"], D, sfb_gran_n=128)
        D_host.copy_(D, non_blocking=True)
        if ev is not None:
            ev[1].record()

    e2e_steps = max(3, min(args.steps, 20))
    e2e_spans = timer.run(e2e_step, 2, e2e_steps)[:, 0]
    serial_ms = max_over_ranks(float(e2e_spans.mean()), world, "cuda")

    # the same steps streamed: step i runs on stream i % 2 with its own device buffers, so its
    # input copies overlap the previous step's GEMM and result read-back (every step still copies
    # all of its inputs in and its result out)
    sets = [{"dev": {key: torch.empty_like(dev[key]) for key in pin},
             "D": torch.empty_like(D), "Dh": torch.empty_like(D_host).pin_memory()} for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]

    def streamed(nsteps):
        cur = torch.cuda.current_stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cur)
        for st in streams:
            st.wait_stream(cur)
        for i in range(nsteps):
            b = sets[i % 2]
            with torch.cuda.stream(streams[i % 2]):
                for key in pin:
                    b["dev"][key].copy_(pin[key], non_blocking=True)
                ops.gemm_fp8_nt(b["dev"]["A"], b["dev"]["sfa"], b["dev"]["B"], b["dev"]["sfb"], b["D"], sfb_gran_n=128)
                b["Dh"].copy_(b["D"], non_blocking=True)
        for st in streams:
            cur.wait_stream(st)
        t1.record(cur)
        t1.synchronize()
        return t0.elapsed_time(t1) / nsteps

    streamed(2)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(streamed(e2e_steps), world, "cuda")
    line["e2e"] = {"value": round(job_flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
                   "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                   "steps": e2e_steps,
                   "api": "ops.gemm_fp8_nt with uint8 UE8M0 scales (packed inside the call), pinned host inputs "
                          "copied in and the bf16 result copied out every step; steps streamed over two CUDA "
                          "streams with two buffer sets",
                   "serial": {"value": round(job_flops / (serial_ms * 1e-3) / 1e12, 2), "ms_per_step": round(serial_ms, 4),
                              "step_time": spread(e2e_spans), "note": "one step at a time on one stream"}}
    del sets

    if gather:
        line["gather_ms"] = spread(spans[:, 2])
    if world == 1 and not args.only_headline and not sharded:
        line["secondary"] = secondary(torch, ops, timer, args, peaks, peak_kind, sampler, sms)
        line["cpu_baseline"] = cpu_baseline(p)
    if ops.device_status() != 0:
        raise RuntimeError("device status after secondary workloads")
    sampler.stop()
    line["clocks_whole_run"] = sampler.window()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _gemm_entry(name, flops, spans, peak, extra=None, dtype=None, sms=None, clocks=None):
    ms = float(np.mean(spans))
    d = {"tflops": round(flops / (ms * 1e-3) / 1e12, 1), "ms": round(ms, 5), "peak_tflops": round(peak, 1),
         "frac": round(flops / (ms * 1e-3) / 1e12 / peak, 4), "time": spread(spans)}
    if dtype is not None:
        d.update(peak_fractions(flops / (ms * 1e-3) / 1e12, dtype, sms, clocks))
    if clocks is not None:
        d["clocks"] = {k: clocks.get(k) for k in ("sm_mhz", "reasons", "samples")}
    if extra:
        d.update(extra)
    return name, d


def secondary(torch, ops, timer, args, peaks, peak_kind, sampler, sms):
    """The other workloads, each timed like the headline (warm-up, L2 flushed before every
    sample, CUDA events around the one call): REPS samples, with their median and p10/p90."""
    reps = max(SECONDARY_REPS, args.steps)
    out = {"peak_source": f"{peak_kind} bf16 burst x nominal dtype ratio", "samples_per_workload": reps}
    bf16_peak = peaks["bf16_tflops"]

    def timed(fn):
        """Per-sample ms of fn and the clocks sampled while it ran."""
        t0 = time.perf_counter()
        spans = timer.run(fn, args.warmup, reps)[:, 0]
        return spans, sampler.window(t0, time.perf_counter())

    def one_call(call):
        def f(ev):
            if ev is not None:
                ev[0].record()
            call()
            if ev is not None:
                ev[1].record()
        return f

    # BF16 dense, same shape
    p = inputs.dense_bf16_problem(M, N, K, seed=2)
    A = torch.from_numpy(p["A"]).cuda().view(torch.bfloat16)
    B = torch.from_numpy(p["B"]).cuda().view(torch.bfloat16)
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    del p
    spans, clk = timed(one_call(lambda: ops.gemm_bf16_nt(A, B, D)))
    tf = gemm_flops(M, N, K) / (float(np.mean(spans)) * 1e-3) / 1e12
    k, v = _gemm_entry("bf16_4096x7168x16384", gemm_flops(M, N, K), spans, bf16_peak,
                       {"vs_pages_431": round(tf / PAGES_BF16_TFLOPS, 3),
                        "traffic": profiled_traffic("gemm_bf16_4096x7168x16384.md")}, "bf16", sms, clk)
    out[k] = v
    del A, B

    # FP4, same shape
    p = inputs.dense_fp4_problem(M, N, K, seed=6)
    d4 = {key: torch.from_numpy(p[key]).cuda() for key in ("A", "sfa", "B", "sfb")}
    sa = ops.transform_sf_ue8m0(d4["sfa"])
    sb = ops.transform_sf_ue8m0(d4["sfb"])
    del p
    spans, clk = timed(one_call(lambda: ops.gemm_fp4_nt(d4["A"], sa, d4["B"], sb, D)))
    k, v = _gemm_entry("fp4_4096x7168x16384", gemm_flops(M, N, K), spans, bf16_peak * NOMINAL_RATIO["fp4"],
                       {"traffic": profiled_traffic("gemm_fp4_4096x7168x16384.md")}, "fp4", sms, clk)
    out[k] = v
    del d4, sa, sb

    # FP8 M sweep at N = K = 7168
    sweep = {}
    for m in (128, 1024, 4096):
        p, dv = fp8_device_problem(torch, m, 7168, 7168, seed=30 + m)
        sa = ops.transform_sf_ue8m0(dv["sfa"])
        sb = ops.transform_sf_ue8m0(dv["sfb"])
        Dm = torch.empty((m, 7168), dtype=torch.bfloat16, device="cuda")
        spans, clk = timed(one_call(lambda dv=dv, sa=sa, sb=sb, Dm=Dm: ops.gemm_fp8_nt(dv["A"], sa, dv["B"], sb, Dm)))
        ms = float(np.mean(spans))
        bytes_min = m * 7168 + 7168 * 7168 + 2 * m * 7168
        fl = gemm_flops(m, 7168, 7168)
        sweep[str(m)] = {"tflops": round(fl / (ms * 1e-3) / 1e12, 1), "ms": round(ms, 5), "time": spread(spans),
                         "frac_tensor": round(fl / (ms * 1e-3) / 1e12 / (bf16_peak * 2), 4),
                         "hbm_gbs_min_bytes": round(bytes_min / (ms * 1e-3) / 1e9, 1),
                         "hbm_frac_min_bytes": round(bytes_min / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                         "plan": ops.gemm_plan("fp8", m, 7168, 7168), "sm_mhz": clk.get("sm_mhz")}
        sweep[str(m)]["traffic"] = profiled_traffic("gemm_fp8_transposed_128x7168x7168.md" if m == 128 else
                                                    f"gemm_fp8_{m}x7168x7168.md")
        del p, dv, sa, sb, Dm
    out["fp8_m_sweep_n7168_k7168"] = sweep

    # M-grouped FP8 MoE workload
    g = inputs.grouped_fp8_problem(32, 32768, 4096, 7168, seed=8)
    dg = {key: torch.from_numpy(g[key]).cuda() for key in ("A", "sfa", "B", "m_indices")}
    sfa_g = ops.transform_sf_ue8m0(dg["sfa"])
    sfb_g = torch.stack([ops.transform_sf_ue8m0(torch.from_numpy(g["sfb"][e]).cuda()) for e in range(32)])
    Dg = torch.empty((g["M"], 4096), dtype=torch.bfloat16, device="cuda")
    spans, clk = timed(one_call(
        lambda: ops.m_grouped_gemm_fp8_nt_contiguous(dg["A"], sfa_g, dg["B"], sfb_g, dg["m_indices"], Dg)))
    fl_valid = gemm_flops(32768, 4096, 7168)
    fl_padded = gemm_flops(g["M"], 4096, 7168)
    k, v = _gemm_entry("grouped_fp8_32x32768x4096x7168", fl_valid, spans, bf16_peak * 2,
                       {"m_total_padded": int(g["M"]),
                        "tflops_incl_padding": round(fl_padded / (float(np.mean(spans)) * 1e-3) / 1e12, 1),
                        "plan": ops.gemm_plan("grouped_fp8", int(g["M"]), 4096, 7168),
                        "traffic": profiled_traffic("gemm_grouped_fp8_32x32768x4096x7168.md")}, "fp8", sms, clk)
    out[k] = v

    # masked grouped (decode-time MoE): 32 experts, slabs of 256 rows, counts uniform in [0, 256]
    # drawn from the seed, N = 4096, K = 7168; every expert with rows streams its whole B
    pm = inputs.masked_fp8_problem(32, 256, 4096, 7168, seed=12)
    dm = {key: torch.from_numpy(pm[key]).cuda() for key in ("A", "sfa", "B", "masked_m")}
    sfa_m = ops.transform_sf_ue8m0(dm["sfa"])
    sfb_m = torch.stack([ops.transform_sf_ue8m0(torch.from_numpy(pm["sfb"][e]).cuda()) for e in range(32)])
    Dm = torch.empty((32, 256, 4096), dtype=torch.bfloat16, device="cuda")
    spans, clk = timed(one_call(
        lambda: ops.m_grouped_gemm_fp8_nt_masked(dm["A"], sfa_m, dm["B"], sfb_m, dm["masked_m"], Dm)))
    ms = float(np.mean(spans))
    rows_valid = int(pm["masked_m"].sum())
    experts_used = int((pm["masked_m"] > 0).sum())
    moved = experts_used * 4096 * 7168 + rows_valid * (7168 + 2 * 4096)  # B of used experts, A and D rows
    k, v = _gemm_entry("masked_fp8_32x256x4096x7168", gemm_flops(rows_valid, 4096, 7168), spans, bf16_peak * 2,
                       {"rows_valid": rows_valid, "gbs_min_bytes": round(moved / (ms * 1e-3) / 1e9, 1),
                        "hbm_frac_min_bytes": round(moved / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                        "traffic": profiled_traffic("gemm_masked_fp8_32x256x4096x7168.md")}, None, sms, clk)
    out[k] = v
    del pm, dm, sfa_m, sfb_m, Dm

    # scale transform alone: the grouped workload's SFA (fp32 scales [M_total, 56]) -> int16 words,
    # the same rows 64 times over in one call (where bandwidth rather than launch latency bounds
    # it), and the FP4 workload's B scales (fp32, one per 32 K: [7168, 512])
    s32 = torch.from_numpy(np.ldexp(np.float32(1), g["sfa"].astype(np.int32) - 127).astype(np.float32)).cuda()
    del g, dg, Dg
    e4 = np.random.default_rng(44).integers(110, 140, size=(N, K // 32)).astype(np.int32)
    s4 = torch.from_numpy(np.ldexp(np.float32(1), e4 - 127).astype(np.float32)).cuda()
    for name, src in (("sf_transform_fp32_36864x56", s32), ("sf_transform_fp32_64x36864x56", s32.repeat(64, 1)),
                      ("sf_transform_fp32_7168x512", s4)):
        w = torch.empty(((src.shape[1] + 1) // 2, ops.sf_ld(src.shape[0])), dtype=torch.int16, device="cuda")
        spans, clk = timed(one_call(lambda src=src, w=w: ops.transform_sf_ue8m0(src, out=w)))
        ms = float(np.mean(spans))
        moved = src.numel() * 4 + w.numel() * 2
        out[name] = {"gbs": round(moved / (ms * 1e-3) / 1e9, 1), "ms": round(ms, 5), "bytes": int(moved),
                     "time": spread(spans), "hbm_peak_gbs": peaks["hbm_gbs"],
                     "frac": round(moved / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "traffic": profiled_traffic(name + ".md"), "sm_mhz": clk.get("sm_mhz")}
        del w
    del s32, s4

    # the quantiser (the step before the GEMM): the headline's A as fp32 in 1x128 blocks and its
    # B as bf16 in 128x128 blocks, values -> E4M3 codes + packed UE8M0 words
    for name, rows, bf16, br in (("quantize_fp8_fp32_4096x16384_1x128", M, False, 1),
                                 ("quantize_fp8_bf16_7168x16384_128x128", N, True, 128)):
        xh = inputs.normal_matrix(rows, K, seed=60 + rows, bf16=bf16)
        x = torch.from_numpy(xh).cuda()
        x = x.view(torch.bfloat16) if bf16 else x
        del xh
        qx, sx = ops.quantize_fp8(x, br)
        spans, clk = timed(one_call(lambda x=x, qx=qx, sx=sx, br=br: ops.quantize_fp8(x, br, q=qx, sf=sx)))
        ms = float(np.mean(spans))
        moved = x.numel() * x.element_size() + qx.numel() + sx.numel() * 2
        out[name] = {"gbs": round(moved / (ms * 1e-3) / 1e9, 1), "ms": round(ms, 5), "bytes": int(moved),
                     "time": spread(spans), "hbm_peak_gbs": peaks["hbm_gbs"],
                     "frac": round(moved / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "traffic": profiled_traffic(name + ".md"), "sm_mhz": clk.get("sm_mhz")}
        del x, qx, sx
    return out


def cpu_baseline(p, budget_s: float = 10.0):
    """The oracle as it stands, on leading rows of the same FP8 problem, for about budget_s."""
    import oracle

    oracle.build()
    rows_done, t_total = 0, 0.0
    chunk = 16
    while t_total < budget_s and rows_done < M:
        r = np.arange(rows_done, min(rows_done + chunk, M), dtype=np.int32)
        t0 = time.perf_counter()
        oracle.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=128, rows=r)
        t_total += time.perf_counter() - t0
        rows_done += len(r)
    return {"value": round(gemm_flops(rows_done, N, K) / t_total / 1e12, 6), "unit": "TFLOPS",
            "cores": oracle.threads(), "kind": "oracle",
            "sample": f"first {rows_done} of {M} rows x all {N} columns of the FP8 {M}x{N}x{K} GEMM "
                      f"({t_total:.1f} s)"}


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return  # the CPU reference runs once, on rank 0
    import oracle

    oracle.build()
    p = inputs.dense_fp8_problem(M, N, K, seed=100)
    # 32 rows a step (about 0.1-0.2 s on the machine's cores): enough rows for every host thread
    rows_per_step = 32

    def step(i):
        r0 = (i * rows_per_step) % M
        oracle.gemm_fp8(p["A"], p["sfa"], p["B"], p["sfb"], gran_n=128,
                        rows=np.arange(r0, r0 + rows_per_step, dtype=np.int32))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = (time.perf_counter() - t0) / args.steps
    value = gemm_flops(rows_per_step, N, K) / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "strong" if getattr(args, "shard", "none") == "n" else "weak",
            "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic",
            "config": workload_config(world, getattr(args, "shard", "none"), getattr(args, "gather", False)),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": oracle.threads(),
                             "kind": "oracle", "sample": f"{rows_per_step} rows x {N} columns per step"},
            "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """Only the named kernel, warm-up + steps times, at the workload's full size (for ncu)."""
    import torch

    from block_scaled_precision_sm_b200 import ops

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    if args.profile == "fp8":
        p, dv = fp8_device_problem(torch, M, N, K, seed=100)
        sa, sb = ops.transform_sf_ue8m0(dv["sfa"]), ops.transform_sf_ue8m0(dv["sfb"])
        D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.gemm_fp8_nt(dv["A"], sa, dv["B"], sb, D)  # noqa: E731
    elif args.profile in ("fp8_m128", "fp8_m1024", "fp8_m4096"):  # the M sweep at N = K = 7168
        m = int(args.profile[5:])
        p, dv = fp8_device_problem(torch, m, 7168, 7168, seed=30 + m)
        sa, sb = ops.transform_sf_ue8m0(dv["sfa"]), ops.transform_sf_ue8m0(dv["sfb"])
        D = torch.empty((m, 7168), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.gemm_fp8_nt(dv["A"], sa, dv["B"], sb, D)  # noqa: E731
    elif args.profile == "bf16":
        p = inputs.dense_bf16_problem(M, N, K, seed=2)
        A = torch.from_numpy(p["A"]).cuda().view(torch.bfloat16)
        B = torch.from_numpy(p["B"]).cuda().view(torch.bfloat16)
        D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.gemm_bf16_nt(A, B, D)  # noqa: E731
    elif args.profile == "fp4":
        p = inputs.dense_fp4_problem(M, N, K, seed=6)
        d4 = {key: torch.from_numpy(p[key]).cuda() for key in ("A", "sfa", "B", "sfb")}
        sa, sb = ops.transform_sf_ue8m0(d4["sfa"]), ops.transform_sf_ue8m0(d4["sfb"])
        D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.gemm_fp4_nt(d4["A"], sa, d4["B"], sb, D)  # noqa: E731
    elif args.profile == "grouped":
        g = inputs.grouped_fp8_problem(32, 32768, 4096, 7168, seed=8)
        dg = {key: torch.from_numpy(g[key]).cuda() for key in ("A", "sfa", "B", "m_indices")}
        sa = ops.transform_sf_ue8m0(dg["sfa"])
        sb = torch.stack([ops.transform_sf_ue8m0(torch.from_numpy(g["sfb"][e]).cuda()) for e in range(32)])
        D = torch.empty((g["M"], 4096), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.m_grouped_gemm_fp8_nt_contiguous(dg["A"], sa, dg["B"], sb, dg["m_indices"], D)  # noqa
    elif args.profile == "masked":
        pm = inputs.masked_fp8_problem(32, 256, 4096, 7168, seed=12)
        dm = {key: torch.from_numpy(pm[key]).cuda() for key in ("A", "sfa", "B", "masked_m")}
        sa = ops.transform_sf_ue8m0(dm["sfa"])
        sb = torch.stack([ops.transform_sf_ue8m0(torch.from_numpy(pm["sfb"][e]).cuda()) for e in range(32)])
        D = torch.empty((32, 256, 4096), dtype=torch.bfloat16, device="cuda")
        fn = lambda: ops.m_grouped_gemm_fp8_nt_masked(dm["A"], sa, dm["B"], sb, dm["masked_m"], D)  # noqa: E731
    elif args.profile in ("quantize_act", "quantize_wgt"):
        act = args.profile == "quantize_act"
        xh = inputs.normal_matrix(M if act else N, K, seed=60 + (M if act else N), bf16=not act)
        x = torch.from_numpy(xh).cuda()
        x = x if act else x.view(torch.bfloat16)
        br = 1 if act else 128
        qx, sx = ops.quantize_fp8(x, br)
        fn = lambda: ops.quantize_fp8(x, br, q=qx, sf=sx)  # noqa: E731
    elif args.profile == "sf_transform_fp4":  # the FP4 workload's B scales, fp32 [7168, 512]
        e4 = np.random.default_rng(44).integers(110, 140, size=(N, K // 32)).astype(np.int32)
        s4 = torch.from_numpy(np.ldexp(np.float32(1), e4 - 127).astype(np.float32)).cuda()
        w = torch.empty((K // 64, ops.sf_ld(N)), dtype=torch.int16, device="cuda")
        fn = lambda: ops.transform_sf_ue8m0(s4, out=w)  # noqa: E731
    else:
        g = inputs.grouped_fp8_problem(32, 32768, 4096, 7168, seed=8)
        s32 = torch.from_numpy(np.ldexp(np.float32(1), g["sfa"].astype(np.int32) - 127).astype(np.float32)).cuda()
        if args.profile == "sf_transform_64x":
            s32 = s32.repeat(64, 1)
        w = torch.empty((28, ops.sf_ld(s32.shape[0])), dtype=torch.int16, device="cuda")
        fn = lambda: ops.transform_sf_ue8m0(s32, out=w)  # noqa: E731
    torch.cuda.synchronize()
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    status = ops.device_status()
    print(json.dumps({"profile": args.profile, "launches": args.warmup + args.steps, "status": status}))
    if status != 0:
        raise SystemExit(1)


def main():
    args = parse()
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
