#!/usr/bin/env python3
"""Benchmark of the W3A16 group-128 decode path on B200.

Workload (one "step"): the Llama-3.1-70B gate_proj shape N=28672, K=8192 with
uint3 codes uniform over 0..7 and lognormal(-4, 0.5) bf16 group scales, run as
three w3a16_gemm calls with batch M = 1, 4 and 16 (x ~ N(0,1) bf16).  Each call
reads a different copy of the weights; five copies (459 MB) rotate, so every
call streams its 91.8 MB of weights from HBM rather than from the 126 MB L2.

Reported: effective HBM GB/s = algorithmic bytes / time, where the algorithmic
bytes of one call are N*K*3/8 (packed) + N*K/128*2 (scales) + M*K*2 (x) +
M*N*2 (y).  `roofline` is the dominant kernel's per-launch figure against the
measured HBM copy bandwidth.  `e2e` is the same metric through the Python API
with every step's x copied from pinned host memory and its y copied back (each
call's y on a second stream as soon as the call ends, largest batch first).
`cpu_baseline` times the CPU oracle on a bounded sample of the same step, on
every host core (OpenMP over rows) and on one.  `configs` adds, on one GPU,
the other configurations: GEMV M=1 4096x4096, down_proj 8192x28672 at M=1 and
8, the Llama-3.1-70B layer at M=1 (7 calls, and 4 row-concatenated calls in
one CUDA graph) and the M=2048 prefill (tensor-core roofline).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs an independent replica (the path does not shard);
value = bytes of all ranks / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W3A16 g128 µs/call and effective HBM GB/s (% of B200 peak) at Llama-70B shapes"
UNIT = "GB/s"
N_ROWS, K_COLS = 28672, 8192
BATCHES = (1, 4, 16)
ROTATE = 5
WORKLOAD = "Llama-3.1-70B gate_proj N=28672 K=8192, W3A16 g128 decode batch M=1,4,16"
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ("w3a16_gemv_b200/csrc/api.cu", "w3a16_gemv_b200/csrc/decode_gemv.cuh",
                  "w3a16_gemv_b200/csrc/decode_split.cuh",
                  "w3a16_gemv_b200/csrc/decode_streamk.cuh", "w3a16_gemv_b200/csrc/decode_tcgen05.cuh",
                  "w3a16_gemv_b200/csrc/prefill_gemm.cuh", "w3a16_gemv_b200/csrc/common.cuh")


def algorithmic_bytes(M: int, N: int, K: int) -> int:
    return N * K * 3 // 8 + N * (K // 128) * 2 + M * K * 2 + M * N * 2


# kernel symbol of each route of w3a16_gemm_route (the names in an ncu launch list)
ROUTE_KERNELS = {
    "decode_split": "w3::dsplit::decode_split_kernel",
    "decode_sk": "w3::decode_sk::decode_sk_kernel",
    "decode": "w3::decode::decode_kernel",
    "decode_tc32": "w3::decode_tc32::decode_tc_kernel",
    "prefill": "w3::prefill::prefill_kernel",
    "prefill_ab": "w3::prefill_ab::prefill_ab_kernel",
    "passes": "16-row decode passes",
}


def route(M: int, N: int, K: int, sms: int) -> str:
    """The kernel route w3a16_gemm takes (asked from the library itself)."""
    from w3a16_gemv_b200 import w3a16_gemm_route

    return w3a16_gemm_route(M, N, K, num_sms=sms)


def kernel_name(M: int, N: int, K: int, sms: int) -> str:
    r = route(M, N, K, sms)
    return f"{ROUTE_KERNELS.get(r, r)} (route {r}, M={M})"


def kernels_per_call(M: int, N: int, K: int, sms: int) -> int:
    """Kernels one w3a16_gemm call launches (asked from the library): the 32-wide tensor-core
    decode is followed by a fix-up kernel when CTA boundaries split its row tiles; every other
    route is one kernel (one per 16-row pass for the passes route)."""
    from w3a16_gemv_b200 import w3a16_gemm_launches

    return w3a16_gemm_launches(M, N, K, num_sms=sms)


def step_bytes() -> int:
    return sum(algorithmic_bytes(m, N_ROWS, K_COLS) for m in BATCHES)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: STREAM-style copy, burst)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier measurement on this pool)"


def sources_sha() -> str:
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_m: int):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_sha") != sources_sha():
        return None
    v = d.get("dram_bytes_per_launch", {}).get(f"M{kernel_m}")
    return float(v) if v is not None else None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []  # (t, sm_mhz, reasons)
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: clocks are reported as unavailable
            self.max_mhz = None

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((time.perf_counter(), mhz, r))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self, t0: float, t1: float):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # timed region shorter than the sampling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:2]
        reasons = 0
        for s in inside:
            reasons |= s[2]
        names = sorted(n for bit, n in self.REASONS.items() if reasons & bit and bit != 0x1)
        return {"sm_mhz": float(statistics.median(s[1] for s in inside)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(inside)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank's measurement all-reduced with MAX (a no-op for one rank).
    Every rank must call it at the same point."""
    if world <= 1:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput per second: the units all replicas processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


# --------------------------------------------------------------------------------------
# CPU oracle (the reported baseline and the reference arm)
# --------------------------------------------------------------------------------------

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def oracle_step_sample(budget_s: float, threads: int | None = None):
    """Time the oracle on slices of the step's weight rows until `budget_s` of wall time is spent.

    threads: None = the plain single-threaded oracle; 0 = its OpenMP variant on every core (rows
    spread over threads, each element the same k-ordered fp64 sum).
    Returns (GB/s in the metric's unit, seconds, rows, threads used, description)."""
    import oracle
    from w3a16_gemv_b200.inputs import make_problem

    orc = oracle.get()
    used = 1 if threads is None else (threads or orc.max_threads())
    rows_per_chunk = 256 * used
    p = make_problem(max(BATCHES), min(rows_per_chunk, N_ROWS), K_COLS, "uniform8", "lognormal", "normal", seed=0)
    packed = orc.pack(p.codes)
    done_rows, spent = 0, 0.0
    while spent < budget_s and done_rows < N_ROWS:
        t0 = time.perf_counter()
        for m in BATCHES:
            orc.gemm_f64(p.x_bf16[:m], packed, p.scales_bf16, threads=threads)
        spent += time.perf_counter() - t0
        done_rows += p.N
    # bytes of the sampled rows in the metric's accounting (weights + the x/y share)
    frac = done_rows / N_ROWS
    nbytes = step_bytes() * frac
    how = "plain C, one thread" if threads is None else f"plain C with OpenMP over rows, {used} threads"
    desc = (f"oracle_gemm_f64 ({how}) for M=1,4,16 over K=8192 on {done_rows} weight rows "
            f"(a {p.N}-row slice of the seeded workload, repeated; {frac:.2%} of one step's rows), "
            f"GB/s = the step's algorithmic bytes scaled by rows / wall seconds; CPU: {cpu_model()}")
    return nbytes / spent / 1e9, spent, done_rows, used, desc


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    per_step = []
    # keep the whole run within a few minutes whatever --steps/--warmup are
    budget = max(0.2, min(args.ref_budget, 150.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step_sample(min(0.5, budget), threads=0)
    desc, used = None, 1
    for _ in range(args.steps):
        gbs, spent, rows, used, desc = oracle_step_sample(budget, threads=0)
        per_step.append((gbs, spent))
    value = statistics.median(g for g, _ in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(1e3 * s for _, s in per_step), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle", "sample": desc,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------

def measured_tensor_peak(sustained: bool = False):
    """The measured cuBLAS bf16 peak: the burst figure, or with `sustained` the figure of a
    seconds-long back-to-back loop under the power cap (the right one for a long timed run)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(path) as f:
            d = json.load(f)
        kind = "back to back for seconds, sustained" if sustained else "burst"
        return float(d[key]), f"measured (MEASURED_PEAKS.json {key}: cuBLAS bf16 GEMM, {kind})"
    except (OSError, KeyError, ValueError):
        if sustained:
            return 1400.0, "fallback (1.4 PFLOP/s sustained, earlier measurement on this pool)"
        return 1590.0, "fallback (1.59 PFLOP/s earlier measurement on this pool)"


def _gpu_setup(world: int, local: int):
    import torch

    from w3a16_gemv_b200 import build as wbuild

    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if not os.path.exists(wbuild.LIB):
        wbuild.build()
    return dev


def measure_prefill(M: int, steps: int, warmup: int, dev, world: int = 1, sampler=None) -> dict:
    """y = x W^T at M x 28672 x 8192 (one call per step), CUDA events around each call."""
    import torch

    from w3a16_gemv_b200 import w3_check_device_error, w3_pack, w3a16_gemm
    from w3a16_gemv_b200.inputs import make_problem

    N, K = N_ROWS, K_COLS
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    p = make_problem(M, N, K, "uniform8", "lognormal", "normal", seed=0)
    packed = w3_pack(torch.from_numpy(p.codes).to(dev))
    scales = torch.from_numpy(p.scales_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    x = torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        w3a16_gemm(x, packed, scales, out=y)
    torch.cuda.synchronize()
    w3_check_device_error()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(steps):
        ev[i][0].record(stream)
        w3a16_gemm(x, packed, scales, out=y)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    w3_check_device_error()
    per_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(ev[0][0].elapsed_time(ev[-1][1]), world, dev)
    flop = 2.0 * M * N * K
    # a timed region of half a second or more runs the tensor cores under the power cap: compare with
    # the sustained figure; a short one with the burst figure
    peak, src = measured_tensor_peak(sustained=total_ms >= 500.0)
    achieved = flop / (statistics.mean(per_ms) * 1e-3) / 1e12
    rec = {
        "workload": f"prefill M={M} N={N} K={K} (Llama-3.1-70B gate_proj), codes uniform 0..7, "
                    "scales bf16 lognormal(-4, 0.5), x bf16 N(0,1)",
        "M": M, "N": N, "K": K, "steps": steps, "total_ms": total_ms,
        "us_per_call": 1e3 * statistics.median(per_ms), "us_mean": 1e3 * statistics.mean(per_ms),
        "TFLOP/s": job_throughput(flop * steps, world, total_ms) / 1e12,
        "GB/s": algorithmic_bytes(M, N, K) / (statistics.mean(per_ms) * 1e-3) / 1e9,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": kernel_name(M, N, K, sms),
                     "peak_source": src, "frac_of_nominal_2250": achieved / 2250.0},
        "l2": f"inputs larger than L2 (x {M * K * 2 / 1e6:.1f} MB + weights {N * K * 3 / 8e6:.1f} MB"
              f" + y {M * N * 2 / 1e6:.1f} MB)",
    }
    if sampler is not None:
        rec["clocks"] = sampler.summary(w0, w1)
    return rec


def run_prefill(args):
    """Prefill workload: y = x W^T at M (default 2048), N=28672, K=8192 (one call per step)."""
    world, rank, local = dist_setup()
    dev = _gpu_setup(world, local)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.02)
    rec = measure_prefill(args.prefill_m, args.steps, args.warmup, dev, world, sampler)
    sampler.stop()
    M = args.prefill_m
    line = {
        "metric": f"W3A16 g128 prefill GEMM TFLOP/s (M={M}, Llama-70B gate_proj)", "value": rec["TFLOP/s"],
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": rec["total_ms"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": rec["workload"], "M": M, "N": N_ROWS, "K": K_COLS, "l2": rec["l2"]},
        "us_per_call": rec["us_per_call"], "roofline": rec["roofline"], "gpu_launches": args.steps,
        "clocks": rec.get("clocks"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch_dist_done()
    return 0


def torch_dist_done():
    import torch

    torch.distributed.destroy_process_group()


SWEEPS = {
    # name: (description, workload names from w3a16_gemv_b200.inputs.workloads())
    "gemv4096": ("W3A16 GEMV M=1 N=4096 K=4096, codes uniform over 2..6, scales |N(0,0.02)|+1e-4",
                 ("gemv_4096_m1",)),
    "down": ("Llama-3.1-70B down_proj N=8192 K=28672 at M=1 and 8, GSQ 5-level codes, x with 1% outliers x20",
             ("down_8192x28672_m1", "down_8192x28672_m8")),
    "layer": ("Llama-3.1-70B layer at M=1: q, k, v, o, gate, up, down projections, codes uniform 0..7",
              ("layer_q_proj_m1", "layer_k_proj_m1", "layer_v_proj_m1", "layer_o_proj_m1",
               "layer_gate_proj_m1", "layer_up_proj_m1", "layer_down_proj_m1")),
}


def _graph_us(calls_of_copy, copies: int, reps: int, stream) -> float:
    """Device time per call: one CUDA graph holding the call on every weight copy, replayed."""
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(copies):
            calls_of_copy(r)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * copies)
    del g
    return us


def measure_sweep(name: str, steps: int, warmup: int, dev, sampler=None) -> dict:
    """Per-call timing of one of the other decode configurations (one GPU): each call's weights
    rotate among enough copies that every call streams them from HBM; device time per call from a
    replayed CUDA graph of the call over its copies; for the layer sweep, also one CUDA graph of the
    seven calls and the 4-call fused layer."""
    import torch

    from w3a16_gemv_b200 import w3_check_device_error, w3_pack, w3a16_gemm
    from w3a16_gemv_b200.inputs import workloads

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    desc, names = SWEEPS[name]
    wls = [workloads()[n] for n in names]
    pass_bytes = sum(algorithmic_bytes(0, w.N, w.K) for w in wls)
    copies = max(2, -(-3 * 126_000_000 // pass_bytes))  # more than three L2 sizes in rotation
    calls = []
    for w in wls:
        p = w.problem()
        packed = w3_pack(torch.from_numpy(p.codes).to(dev))
        sc = torch.from_numpy(p.scales_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
        x = torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
        calls.append({"w": w, "packs": [packed] + [packed.clone() for _ in range(copies - 1)],
                      "scales": [sc] + [sc.clone() for _ in range(copies - 1)], "x": x,
                      "y": torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)})
    stream = torch.cuda.current_stream()

    def one_pass(i, ev=None):
        for j, c in enumerate(calls):
            r = i % copies
            if ev is not None:
                ev[j][0].record(stream)
            w3a16_gemm(c["x"], c["packs"][r], c["scales"][r], out=c["y"])
            if ev is not None:
                ev[j][1].record(stream)

    for i in range(warmup):
        one_pass(i)
    torch.cuda.synchronize()
    w3_check_device_error()
    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in calls]
              for _ in range(steps)]
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(steps):
        one_pass(warmup + i, events[i])
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    w3_check_device_error()
    reps = max(3, steps // copies)
    graph_us = [_graph_us(lambda r, c=c: w3a16_gemm(c["x"], c["packs"][r], c["scales"][r], out=c["y"]),
                          copies, reps, stream) for c in calls]
    w3_check_device_error()
    peak, peak_src = measured_peak()
    out_calls, total_us, total_bytes = [], 0.0, 0
    for j, c in enumerate(calls):
        w = c["w"]
        ts = np.array([events[i][j][0].elapsed_time(events[i][j][1]) for i in range(steps)]) * 1e3
        med = float(np.median(ts))
        b = algorithmic_bytes(w.M, w.N, w.K)
        total_us += med
        total_bytes += b
        gu = graph_us[j]
        out_calls.append({"name": w.name, "M": w.M, "N": w.N, "K": w.K, "kernel": kernel_name(w.M, w.N, w.K, sms),
                          "us_median": med, "us_p10": float(np.percentile(ts, 10)),
                          "us_p90": float(np.percentile(ts, 90)), "us_device_graph": gu,
                          "GB/s": b / (gu * 1e-6) / 1e9, "frac_of_peak": b / (gu * 1e-6) / 1e9 / peak,
                          "TFLOP/s": 2.0 * w.M * w.N * w.K / (gu * 1e-6) / 1e12})
    rec = {
        "workload": desc, "calls_list": list(names), "GB/s": total_bytes / (sum(graph_us) * 1e-6) / 1e9,
        "frac_of_peak": total_bytes / (sum(graph_us) * 1e-6) / 1e9 / peak,
        "sum_of_median_us": total_us, "sum_of_device_us": sum(graph_us), "steps": steps,
        "l2": f"inputs larger than L2: {copies} rotating copies of every call's weights "
              f"({copies * pass_bytes / 1e6:.0f} MB)",
        "timing": "us_median/p10/p90: CUDA events around each call (include host launch overhead when the "
                  "kernel is shorter than it); us_device_graph and GB/s: one CUDA graph of the call on every "
                  "weight copy, replayed, time per call",
        "calls": out_calls, "peak": peak, "peak_source": peak_src,
    }
    if sampler is not None:
        rec["clocks"] = sampler.summary(w0, w1)
    if name == "layer":
        # one CUDA graph of the seven calls on fixed copies, replayed
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            one_pass(0)  # warm the side stream outside the capture
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            one_pass(0)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        w3_check_device_error()
        g_us = a.elapsed_time(b) * 1e3 / steps
        rec["cuda_graph"] = {"us_per_replay": g_us, "GB/s": total_bytes / (g_us * 1e-6) / 1e9,
                             "note": "weights of one copy, 7 calls per replay (L2 holds part of them)"}
        del g
        rec["fused"] = fused_layer(calls, copies, steps, stream, total_bytes)
    return rec


def run_sweep(args):
    import torch

    world, rank, local = dist_setup()
    if rank != 0:
        return 0
    torch.cuda.set_device(local)
    dev = _gpu_setup(1, local)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.02)
    rec = measure_sweep(args.workload, args.steps, args.warmup, dev, sampler)
    sampler.stop()
    line = {
        "metric": METRIC, "value": rec["GB/s"], "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["sum_of_device_us"] / 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": rec["workload"], "calls": rec["calls_list"], "l2": rec["l2"]},
    }
    line.update({k: v for k, v in rec.items() if k not in ("workload", "calls_list", "l2", "GB/s")})
    print(json.dumps(line), flush=True)
    return 0


def fused_layer(calls, copies, steps, stream, total_bytes):
    """The same layer as 4 calls: q, k, v and gate, up concatenated along N (rows of the format
    are independent, so a row-concatenated packed/scales pair is one weight), o and down alone.
    Device time of each call from graph replays over its copies, and one graph of the 4 calls."""
    import torch

    from w3a16_gemv_b200 import w3_check_device_error, w3a16_gemm

    by = {c["w"].name: c for c in calls}

    def cat(names):
        cs = [by[n] for n in names]
        return {"name": "+".join(n.split("_")[1] for n in names), "M": 1,
                "N": sum(c["w"].N for c in cs), "K": cs[0]["w"].K, "x": cs[0]["x"],
                "packs": [torch.cat([c["packs"][r] for c in cs]) for r in range(copies)],
                "scales": [torch.cat([c["scales"][r] for c in cs]) for r in range(copies)]}

    fcalls = [cat(["layer_q_proj_m1", "layer_k_proj_m1", "layer_v_proj_m1"]), cat(["layer_o_proj_m1"]),
              cat(["layer_gate_proj_m1", "layer_up_proj_m1"]), cat(["layer_down_proj_m1"])]
    for c in fcalls:
        c["y"] = torch.empty((1, c["N"]), dtype=torch.bfloat16, device=c["x"].device)
    reps = max(3, steps // copies)
    out = []
    for c in fcalls:
        us = _graph_us(lambda r, c=c: w3a16_gemm(c["x"], c["packs"][r], c["scales"][r], out=c["y"]), copies, reps,
                       stream)
        byt = algorithmic_bytes(1, c["N"], c["K"])
        out.append({"name": c["name"], "N": c["N"], "K": c["K"], "us_device_graph": us,
                    "GB/s": byt / (us * 1e-6) / 1e9})
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in fcalls:
            w3a16_gemm(c["x"], c["packs"][0], c["scales"][0], out=c["y"])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    w3_check_device_error()
    g_us = a.elapsed_time(b) * 1e3 / steps
    del g
    return {"calls": out, "sum_of_device_us": sum(c["us_device_graph"] for c in out),
            "cuda_graph_us_per_replay": g_us, "GB/s": total_bytes / (g_us * 1e-6) / 1e9}


def measure_native_step(p, steps: int, dev) -> dict:
    """The headline decode step (gate_proj, M = 1, 4, 16) on the kernel-native block order of the
    same weights (w3_native_from_packed, done once, outside the timed region): the step back to
    back, and each call back to back on its own, device time with CUDA events."""
    import torch

    from w3a16_gemv_b200 import w3_check_device_error, w3_native_from_packed, w3_pack, w3a16_gemm_native

    natives = [w3_native_from_packed(w3_pack(torch.from_numpy(p.codes).to(dev)), K_COLS)]
    natives += [natives[0].clone() for _ in range(ROTATE - 1)]
    sc0 = torch.from_numpy(p.scales_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    scs = [sc0] + [sc0.clone() for _ in range(ROTATE - 1)]
    x_all = torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    xs = {m: x_all[:m].contiguous() for m in BATCHES}
    ys = {m: torch.empty((m, N_ROWS), dtype=torch.bfloat16, device=dev) for m in BATCHES}
    stream = torch.cuda.current_stream()
    peak, _ = measured_peak()

    def call(i, j, m):
        c = (i * len(BATCHES) + j) % ROTATE
        w3a16_gemm_native(xs[m], natives[c], scs[c], N_ROWS, out=ys[m])

    for i in range(ROTATE):
        for j, m in enumerate(BATCHES):
            call(i, j, m)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        for j, m in enumerate(BATCHES):
            call(i, j, m)
    b.record(stream)
    torch.cuda.synchronize()
    step_ms = a.elapsed_time(b) / steps
    calls = []
    for j, m in enumerate(BATCHES):
        a.record(stream)
        for i in range(steps):
            call(i, j, m)
        b.record(stream)
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / steps
        byt = algorithmic_bytes(m, N_ROWS, K_COLS)
        calls.append({"M": m, "us_mean": us, "GB/s": byt / (us * 1e-6) / 1e9,
                      "frac_of_peak": byt / (us * 1e-6) / 1e9 / peak})
    w3_check_device_error()
    return {"workload": WORKLOAD + ", weights in the kernel-native block order (w3a16_gemm_native)",
            "GB/s": step_bytes() / (step_ms * 1e-3) / 1e9, "ms_per_step": step_ms, "steps": steps, "calls": calls}


def run_gpu(args):
    import torch

    from w3a16_gemv_b200 import w3_check_device_error, w3_pack, w3a16_gemm
    from w3a16_gemv_b200.inputs import make_problem

    world, rank, local = dist_setup()
    dev = _gpu_setup(world, local)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    # ---- inputs: seeded, drawn on the host, packed on the device by w3_pack ----
    p = make_problem(max(BATCHES), N_ROWS, K_COLS, "uniform8", "lognormal", "normal", seed=0)
    codes_d = torch.from_numpy(p.codes).to(dev)
    packed0 = w3_pack(codes_d)
    del codes_d
    scales0 = torch.from_numpy(p.scales_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    packs = [packed0] + [packed0.clone() for _ in range(ROTATE - 1)]
    scales = [scales0] + [scales0.clone() for _ in range(ROTATE - 1)]
    x_all = torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    xs = {m: x_all[:m].contiguous() for m in BATCHES}
    ys = {m: torch.empty((m, N_ROWS), dtype=torch.bfloat16, device=dev) for m in BATCHES}
    torch.cuda.synchronize()

    calls_per_step = len(BATCHES)
    stream = torch.cuda.current_stream()

    def one_step(i, ev=None):
        for j, m in enumerate(BATCHES):
            c = (i * calls_per_step + j) % ROTATE
            if ev is not None:
                ev[j][0].record(stream)
            w3a16_gemm(xs[m], packs[c], scales[c], out=ys[m])
            if ev is not None:
                ev[j][1].record(stream)

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()
    w3_check_device_error()

    # ---- timed region: K steps back to back, barrier + synchronize on both sides.  Nothing is
    #      recorded between the calls, so a call's kernel may start its set-up while the previous
    #      one finishes (programmatic dependent launch), as in a model's decode step ----
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.02)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    t_start.record(stream)
    for i in range(args.steps):
        one_step(args.warmup + i)
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    w3_check_device_error()
    elapsed_ms = t_start.elapsed_time(t_end)

    # ---- per-call breakdown, two ways (further timed passes, at least 200 calls each):
    #      stream: each call of the step launched back to back on its own (rotating weight copies,
    #        programmatic dependent launch, as in the step), one event pair around the whole run:
    #        the mean launch duration the roofline uses;
    #      isolated: an event pair around every call of the step, which also keeps consecutive
    #        calls from overlapping ----
    brk_steps = max(200, min(args.steps, 500))
    stream_us = {}
    for j, m in enumerate(BATCHES):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(ROTATE):
            w3a16_gemm(xs[m], packs[i], scales[i], out=ys[m])
        a.record(stream)
        for i in range(brk_steps):
            c = (i * calls_per_step + j) % ROTATE
            w3a16_gemm(xs[m], packs[c], scales[c], out=ys[m])
        b.record(stream)
        torch.cuda.synchronize()
        stream_us[m] = a.elapsed_time(b) * 1e3 / brk_steps
    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in BATCHES] for _ in range(brk_steps)]
    for i in range(brk_steps):
        one_step(args.warmup + args.steps + i, events[i])
    torch.cuda.synchronize()
    sampler.stop()
    w3_check_device_error()
    per_call_ms = {m: [events[i][j][0].elapsed_time(events[i][j][1]) for i in range(brk_steps)]
                   for j, m in enumerate(BATCHES)}

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    value = job_throughput(step_bytes() * args.steps, world, elapsed_ms) / 1e9
    ms_per_step = elapsed_ms / args.steps

    # ---- roofline of the dominant kernel (largest share of the step) ----
    peak, peak_src = measured_peak()
    calls = []
    for m in BATCHES:
        us = stream_us[m]
        iso = 1e3 * statistics.mean(per_call_ms[m])
        b = algorithmic_bytes(m, N_ROWS, K_COLS)
        q = np.percentile(np.array(per_call_ms[m]) * 1e3, [10, 90])
        calls.append({"M": m, "kernel": kernel_name(m, N_ROWS, K_COLS, sms), "us_mean": us,
                      "us_isolated_mean": iso, "us_isolated_median": 1e3 * statistics.median(per_call_ms[m]),
                      "us_isolated_p10": float(q[0]), "us_isolated_p90": float(q[1]),
                      "GB/s": b / (us * 1e-6) / 1e9, "TFLOP/s": 2.0 * m * N_ROWS * K_COLS / (us * 1e-6) / 1e12,
                      "frac_of_peak": b / (us * 1e-6) / 1e9 / peak,
                      "frac_of_peak_isolated": b / (iso * 1e-6) / 1e9 / peak, "share": 0.0})
    tot = sum(c["us_mean"] for c in calls)
    for c in calls:
        c["share"] = c["us_mean"] / tot
    dom = max(calls, key=lambda c: c["us_mean"])
    roofline = {"bound": "hbm", "achieved": dom["GB/s"], "peak": peak, "unit": "GB/s",
                "frac": dom["GB/s"] / peak, "traffic": recorded_traffic(dom["M"]),
                "kernel": dom["kernel"],
                "algorithmic_bytes_per_launch": algorithmic_bytes(dom["M"], N_ROWS, K_COLS),
                "launch_time": f"mean over {brk_steps} launches of the call back to back (rotating weight copies, "
                               "programmatic dependent launch as in the step), CUDA events on the launch stream; "
                               "frac_isolated: the same call with an event pair around each launch",
                "frac_isolated": dom["frac_of_peak_isolated"],
                "peak_source": peak_src}

    # ---- end to end through the public API with host buffers ----
    # One pinned host buffer holds the step's inputs (the three batches' rows stacked) and one its
    # outputs.  Per step: one host-to-device copy of every x, the three calls, and each call's y
    # copied back on a second stream as soon as that call ends, so that the copies overlap the
    # calls after it.  The calls run largest batch first (M = 16, 4, 1): the largest y crosses
    # while the other two calls run and only the 57 KB of the M = 1 call is left exposed.  The
    # step ends when the last copy has landed; the next step's inputs are copied only after that.
    e2e_order = tuple(sorted(BATCHES, reverse=True))
    rows = [0]
    for m in e2e_order:
        rows.append(rows[-1] + m)
    x_host = torch.empty((rows[-1], K_COLS), dtype=torch.bfloat16).pin_memory()
    for j, m in enumerate(e2e_order):
        x_host[rows[j]:rows[j + 1]].copy_(xs[m].cpu())
    x_dev = torch.empty((rows[-1], K_COLS), dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty((rows[-1] * N_ROWS,), dtype=torch.bfloat16, device=dev)
    y_host = torch.empty((rows[-1] * N_ROWS,), dtype=torch.bfloat16).pin_memory()
    xd = [x_dev[rows[j]:rows[j + 1]] for j in range(len(e2e_order))]
    yd = [y_dev[rows[j] * N_ROWS:rows[j + 1] * N_ROWS].view(m, N_ROWS) for j, m in enumerate(e2e_order)]
    yh = [y_host[rows[j] * N_ROWS:rows[j + 1] * N_ROWS].view(m, N_ROWS) for j, m in enumerate(e2e_order)]
    copy_stream = torch.cuda.Stream(device=dev)
    call_done = [torch.cuda.Event() for _ in e2e_order]
    e2e_steps = max(1, min(args.steps, 200))

    def e2e_step(i):
        x_dev.copy_(x_host, non_blocking=True)
        for j, m in enumerate(e2e_order):
            c = (i * calls_per_step + j) % ROTATE
            w3a16_gemm(xd[j], packs[c], scales[c], out=yd[j])
            call_done[j].record(stream)
            copy_stream.wait_event(call_done[j])
            with torch.cuda.stream(copy_stream):
                yh[j].copy_(yd[j], non_blocking=True)
        copy_stream.synchronize()

    for i in range(3):
        e2e_step(i)
    e2e_ok = all(torch.equal(yh[j].to(dev), yd[j]) for j in range(len(e2e_order)))
    if world > 1:
        torch.distributed.barrier()
    e0 = time.perf_counter()
    for i in range(e2e_steps):
        e2e_step(i)
    e_ms = (time.perf_counter() - e0) * 1e3
    e_ms = max_over_ranks(e_ms, world, dev)
    e2e = {"value": job_throughput(step_bytes() * e2e_steps, world, e_ms) / 1e9, "unit": UNIT,
           "h2d_bytes_per_step": sum(m * K_COLS * 2 for m in BATCHES),
           "d2h_bytes_per_step": sum(m * N_ROWS * 2 for m in BATCHES),
           "steps": e2e_steps, "ms_per_step": e_ms / e2e_steps,
           "method": "wall clock over the steps; per step one pinned host-to-device copy of every x, the "
                     "calls M = " + ", ".join(str(m) for m in e2e_order) + " through w3a16_gemm, each "
                     "call's y copied to pinned host memory on a second stream as soon as the call ends, "
                     "and a synchronisation on the last copy",
           "host_copy_matches_device": e2e_ok}

    clocks = sampler.summary(w0, w1)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": list(BATCHES), "N": N_ROWS, "K": K_COLS,
                   "codes": "uniform 0..7", "scales": "bf16 lognormal(-4, 0.5)", "x": "bf16 N(0,1)",
                   "l2": f"inputs larger than L2: {ROTATE} rotating weight copies "
                         f"({ROTATE * algorithmic_bytes(0, N_ROWS, K_COLS) / 1e6:.0f} MB > 126 MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "step_bytes": step_bytes()},
        "us_per_call": {f"M{c['M']}": c["us_mean"] for c in calls},
        "calls": calls,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps * sum(kernels_per_call(m, N_ROWS, K_COLS, sms) for m in BATCHES),
        "per_call_timing": f"calls[].us_mean: each call launched {brk_steps} times back to back (rotating weight "
                           "copies, programmatic dependent launch), CUDA events around the run; us_isolated_*: "
                           "an event pair around every call; value: the K steps back to back",
        "clocks": clocks,
    }
    del packs, scales, x_all, xs, ys, x_dev, y_dev
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_configs:
        # the other configurations, each on its own inputs (one GPU; device time per call)
        cs = ClockSampler(local)
        cs.start()
        time.sleep(0.02)
        configs = {"1_gemv_4096": measure_sweep("gemv4096", 50, 5, dev, cs),
                   "2_gate_decode": {"workload": WORKLOAD, "see": "value, calls, roofline of this line"},
                   "2n_gate_decode_native": measure_native_step(p, brk_steps, dev),
                   "3_down_proj": measure_sweep("down", 50, 5, dev, cs),
                   "4_layer": measure_sweep("layer", 50, 5, dev, cs),
                   "5_prefill_2048": measure_prefill(2048, 20, 3, dev, 1, cs)}
        cs.stop()
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs1, spent1, rows1, _, desc1 = oracle_step_sample(args.cpu_budget / 2)
        gbsn, spentn, rowsn, used, descn = oracle_step_sample(args.cpu_budget / 2, threads=0)
        line["cpu_baseline"] = {"value": gbsn, "unit": UNIT, "cores": used, "kind": "oracle", "sample": descn,
                                "seconds": spentn, "cpu_model": cpu_model(), "os_cpu_count": os.cpu_count(),
                                "single_core": {"value": gbs1, "unit": UNIT, "cores": 1, "sample": desc1,
                                                "seconds": spent1}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch_dist_done()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of CPU oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=3.0, help="seconds of oracle work per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations (GEMV 4096, down_proj, 70B layer, M=2048 prefill)")
    ap.add_argument("--prefill-m", type=int, default=2048, help="batch rows of the prefill workload (M > 32)")
    ap.add_argument("--workload", choices=("gate_decode", "prefill") + tuple(SWEEPS), default="gate_decode",
                    help="gate_decode: the headline decode step (default); prefill: M=2048 tensor-core GEMM; "
                         "gemv4096, down, layer: per-call timings of the other decode configurations")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "prefill":
        return run_prefill(args)
    if args.workload in SWEEPS:
        return run_sweep(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
