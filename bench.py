"""Benchmark: exact Lloyd k-means iterations per second on B200.

One step = one pass of the whole hot path on the embedding workload
(N = 1,048,576 points, D = 128, fp16, K = 1,024 centroids; the workload the
headline metric is quoted on):

    fk_prepare_centroids  (round fp32 centroids to fp16, bias -|c|^2/2)
    fk_assign_prepared    (tcgen05 FlashAssign: distances + online argmin,
                           then the exact re-decision of near-ties)
    fk_update             (sort-inverse update: radix sort, segment offsets,
                           segmented sums, divide)

all through the C ABI, inputs resident in HBM (X = 256 MiB, larger than the
126 MB L2, so no flush is needed between steps); |x|^2 of the points is
prepared once (fk_prepare_points), as X does not change between iterations.

On one GPU the line also carries "workloads": the same measurement of the
other configured workloads (tiny fp32, batched bf16, Zipf bf16) and the
out-of-core one at 2^27 rows (--ooc-rows-all), each with its own rooflines
against the measured and the spec peaks, its CPU baseline and its clocks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--no-e2e] [--no-cpu] [--no-all]
                    [--ooc-rows R] [--ooc-rows-all R]

--workload ooc_f16 runs the out-of-core workload instead (one GPU): X in
pinned host memory, streamed through fk_lloyd_ooc in the configured 64 Mi-row
chunks, --ooc-rows rows (the configured 10^9 rows need 256 GB of pinned host
memory, more than the host has).

Prints one JSON line (rank 0).  Multi-GPU runs are replicas: every rank runs
its own copy of the workload, there is no collective on the data path, the
time is the max over ranks and the value is the sum of all ranks' steps
divided by it ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "k-means Lloyd iter/s; assign TFLOP/s & update GB/s as % of B200 roofline"
UNIT = "iter/s"
# FP32 lanes per SM and the maximum SM clock of a B200 (clocks.max.sm), for the
# roofline of the fp32 CUDA-core assign kernel
FP32_LANES_PER_SM = 128
SM_MAX_GHZ = 1.965
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------- rank helpers --
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(steps_per_rank: int, elapsed_ms: float, world: int, device=None):
    """Whole-job throughput: all ranks' steps over the slowest rank's time."""
    t_max = max_over_ranks(elapsed_ms, world, device)
    units = sum_over_ranks(float(steps_per_rank), world, device)
    return units / (t_max / 1e3), t_max


# ----------------------------------------------------------------- peaks --
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled in the background."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index
        self.period = period_ms
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self._t:
                self._t.join(timeout=2)

    def summary(self, t0: float, t1: float):
        def parse(r):
            f = [x.strip() for x in r.split(",")]
            try:
                return {"sm": float(f[1]), "max": float(f[2]), "active": f[4],
                        "hw_slowdown": f[5], "hw_thermal_slowdown": f[6],
                        "sw_thermal_slowdown": f[7], "sw_power_cap": f[8]}
            except (ValueError, IndexError):
                return None
        inside = [parse(r) for (t, r) in self.rows if t0 <= t <= t1]
        inside = [x for x in inside if x]
        window = "timed"
        if not inside:  # region shorter than the sampling period: nearest samples
            near = sorted(self.rows, key=lambda tr: min(abs(tr[0] - t0), abs(tr[0] - t1)))[:3]
            inside = [x for x in (parse(r) for _, r in near) if x]
            window = "nearest to timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = sorted({k for x in inside for k in ("hw_slowdown", "hw_thermal_slowdown",
                                                       "sw_thermal_slowdown", "sw_power_cap")
                          if x[k].lower() == "active"})
        return {"sm_mhz": statistics.median(x["sm"] for x in inside),
                "sm_max_mhz": max(x["max"] for x in inside), "reasons": reasons,
                "samples": len(inside), "window": window}


# --------------------------------------------------------- profile data --
def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("assign_tc.cu", "tc_argmin.cuh", "fk_common.cuh"):
        with open(os.path.join(ROOT, "distance_argmin_flashassign_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the assign kernel from the committed ncu
    summary, or None when absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", f"assign_tc_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        p = json.load(f)
    if p.get("kernel_source_hash") != kernel_source_hash():
        return None
    return p.get("dram_bytes_per_launch")


# ------------------------------------------------------------ CPU oracle --
def oracle_throughput(X64, C64, dtype: str, N_full: int, budget_s: float):
    """Time the oracle's Lloyd step on the first rows of the workload (all K
    centroids) for about ``budget_s`` seconds and scale linearly in N to
    iterations per second of the full workload.  When the whole workload fits
    the budget, whole steps are repeated instead."""
    import oracle
    lib = oracle.load()
    n = min(4096, X64.shape[0])
    t = time.perf_counter()
    oracle.lloyd_step(X64[:n], C64, dtype, lib)
    per_row = (time.perf_counter() - t) / n
    n = int(max(n, min(X64.shape[0], budget_s / max(per_row, 1e-9))))
    reps = max(1, int(budget_s / max(per_row * n, 1e-9))) if n == X64.shape[0] else 1
    t = time.perf_counter()
    for _ in range(reps):
        oracle.lloyd_step(X64[:n], C64, dtype, lib)
    dt = time.perf_counter() - t
    return reps * n / (N_full * dt), n, reps, dt, oracle.num_threads()


# ------------------------------------------------------------- workloads --
def build_inputs(name: str, device, seed: int, rows: int = 0):
    """The configured workload `name`; "embed_f32" is the embedding recipe in
    fp32 (the fp32 tensor-core case, not a configured workload)."""
    import workloads
    base, over = (("embed_f16", {"dtype": "f32"}) if name == "embed_f32" else (name, {}))
    if rows:
        over["N"] = rows
    s = workloads.spec(base, **over)
    w = workloads.make(s, seed=seed, device=device)
    return s, w


# Spec peaks of a B200 (the stricter denominators, reported next to the
# measured ones): dense fp16/bf16 tensor throughput and HBM3e bandwidth.
SPEC_P16_TFLOPS = 2250.0
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 / bf16 rate
SFU_EX2_PER_SM_CLK = 16     # ex2.approx per SM per clock (4 per sub-partition)
SPEC_HBM_GBS = 8000.0


def measure(args, name: str, fk, dev, world: int, rank: int, steps: int, warmup: int, cpu_budget: float,
            seed: int):
    """Time `steps` Lloyd iterations of workload `name` resident in HBM: one
    step = fk_prepare_centroids + fk_assign_prepared (the assignment kernel
    and the exact re-decision of near-ties) + fk_update, all through the C
    ABI, with |x|^2 prepared once (X does not change between iterations).
    Returns the workload's JSON fields and the raw timings."""
    import torch
    s, w = build_inputs(name, dev, seed, getattr(args, "rows", 0) if name == args.workload else 0)
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[s.dtype]
    X = w.X
    B, N, D, K = s.B, s.N, s.D, s.K
    C = w.C0.clone()
    C_dt, bias = fk.fk_prepare_centroids(C, dt)
    xnorm = fk.fk_prepare_points(X) if dt != torch.float32 else None
    labels = torch.empty(((B, N) if B > 1 else (N,)), dtype=torch.int32, device=dev)
    counts = torch.empty(((B, K) if B > 1 else (K,)), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        fk.fk_prepare_centroids(C, dt, C_dt, bias)
        if ev:
            ev[0].record(stream)
        fk.fk_assign_prepared(X, C_dt, bias, labels, xnorm=xnorm)
        if ev:
            ev[1].record(stream)
        fk.fk_update(X, labels, C, counts)
        if ev:
            ev[2].record(stream)

    for _ in range(warmup):
        step()
    fk.fk_sync()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)  # let the sampler start before the timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    n0 = fk.fk_launch_count()
    w0 = time.time()
    t_start.record(stream)
    for i in range(steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    launches = fk.fk_launch_count() - n0
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    fk.fk_sync()
    elapsed = t_start.elapsed_time(t_end)
    t_assign = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_update = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    value, t_max = aggregate(steps, elapsed, world, dev)
    peaks, peak_kind = load_peaks()
    flops = 2.0 * B * N * K * D
    es = s.bytes_per_elem
    assign_bytes = B * (N * D * es + K * D * es + 32 * K + 8 * N)
    upd_bytes = B * (N * D * es + 4 * N + K * (4 * D + 4))
    tflops = flops / (t_assign * 1e-3) / 1e12
    gbs = upd_bytes / (t_update * 1e-3) / 1e9
    stage = "assignment stage: assign kernel + exact near-tie re-decision kernel"
    if s.dtype == "f32" and fk.fk_assign_path(N, D, torch.float32, K) == 1:
        # fp32 on the tensor cores as three tf32 passes: the tensor work is 3 x
        # 2NKD, against the tf32 dense peak (the measured bf16 burst peak times
        # the nominal tf32 / bf16 dense ratio, 1.1 / 2.25)
        tf32_peak = peaks["bf16_tflops"] * TF32_PER_BF16
        work = 3.0 * flops
        tf = work / (t_assign * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "assign_tf32_kernel (three tf32 passes)",
                    "stage": stage + " + the hi/lo split of X and C", "achieved": round(tf, 2),
                    "peak": round(tf32_peak, 1), "unit": "TFLOP/s", "frac": round(tf / tf32_peak, 4),
                    "peak_kind": f"{peak_kind} bf16 burst x 1.1/2.25 (nominal tf32/bf16 dense ratio)",
                    "fp32_equivalent_tflops": round(tflops, 2), "traffic": None,
                    "ms_per_launch": round(t_assign, 5), "algorithmic_flops_per_launch": flops,
                    "tensor_flops_per_launch": work}
    elif s.dtype == "f32":
        # fp32 on the CUDA-core kernel: bound by the FP32 FMA pipes, whose
        # peak is derived from the unit counts and the maximum SM clock
        props = torch.cuda.get_device_properties(dev)
        fp32_peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * SM_MAX_GHZ / 1e3
        roofline = {"bound": "alu", "kernel": "assign_simt_kernel", "stage": stage, "achieved": round(tflops, 3),
                    "peak": round(fp32_peak, 1), "unit": "TFLOP/s", "frac": round(tflops / fp32_peak, 4),
                    "peak_kind": f"fp32 FMA: {props.multi_processor_count} SMs x {FP32_LANES_PER_SM} lanes x "
                                 f"2 flop x {SM_MAX_GHZ} GHz (derived from unit counts and clock)",
                    "traffic": None, "ms_per_launch": round(t_assign, 5), "algorithmic_flops_per_launch": flops}
    else:
        ai = flops / assign_bytes
        peak_meas = min(peaks["bf16_tflops"], ai * peaks["hbm_gbs"] / 1e3)
        peak_spec = min(SPEC_P16_TFLOPS, ai * SPEC_HBM_GBS / 1e3)
        bound = "tensor" if peak_meas >= peaks["bf16_tflops"] else "hbm"
        roofline = {"bound": bound, "kernel": "assign_tc_kernel", "stage": stage, "achieved": round(tflops, 2),
                    "peak": round(peak_meas, 1), "unit": "TFLOP/s", "frac": round(tflops / peak_meas, 4),
                    "peak_kind": (f"{peak_kind} bf16 burst (fp16 = bf16 dense rate)" if bound == "tensor" else
                                  f"arithmetic intensity {ai:.0f} flop/B x {peak_kind} copy bandwidth "
                                  "(below the tensor peak)"),
                    "peak_spec": round(peak_spec, 1), "frac_spec": round(tflops / peak_spec, 4),
                    "traffic": profiled_traffic(name), "ms_per_launch": round(t_assign, 5),
                    "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": assign_bytes}
    roofline_update = {"bound": "hbm", "kernels": "fk_update (sort, offsets, segsum, finalize)",
                       "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": f"{peak_kind} copy",
                       "peak_spec": SPEC_HBM_GBS, "frac_spec": round(gbs / SPEC_HBM_GBS, 4),
                       "ms_per_call": round(t_update, 5), "algorithmic_bytes_per_call": upd_bytes}
    out = {"value": round(value, 3), "unit": UNIT, "ms_per_step": round(t_max / steps, 5), "steps": steps,
           "warmup": warmup,
           "config": {"workload": name, "N": N, "D": D, "K": K, "B": B, "dtype": s.dtype,
                      "iterations_configured": s.iters,
                      "step": "one Lloyd iteration: prepare centroids + assign + update",
                      "l2": "inputs larger than L2 (X is %d MiB)" % (B * N * D * es >> 20)},
           "roofline": roofline, "roofline_update": roofline_update, "gpu_launches": launches,
           "clocks": clocks.summary(w0, w1)}
    if rank == 0 and world == 1 and cpu_budget > 0:
        X64 = X.double().cpu().numpy() if B == 1 else X[0].double().cpu().numpy()
        C64 = w.C0.double().cpu().numpy() if B == 1 else w.C0[0].double().cpu().numpy()
        v, n, reps, secs, cores = oracle_throughput(X64, C64, s.dtype, N * B, cpu_budget)
        out["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x {n} of {N * B} rows against all {K} centroids, one Lloyd "
                                         f"step each ({secs:.1f} s in all), scaled linearly in N"}
    return out, s, w


def measure_gauss(args, fk, dev, steps: int, warmup: int):
    """Weighted Gauss sums on the embedding workload's points: G[i] = sum_k
    w_k exp(-beta |x_i - c_k|^2) over its K = 1,024 initial centroids,
    positive weights, beta = 2 (the rows are unit vectors).  One call =
    the bias prep and the tensor-core pass (fp32 accumulation, running
    log-sum-exp)."""
    import torch
    s, w = build_inputs("embed_f16", dev, 0)
    X, C = w.X, w.C0.to(torch.float16)
    N, D, K = s.N, s.D, s.K
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    wt = torch.rand(K, generator=g, device=dev) + 0.5
    G = torch.empty(N, device=dev)
    logG = torch.empty(N, device=dev)
    for _ in range(warmup):
        fk.fk_gauss_sum(X, C, 2.0, w=wt, G=G, logG=logG)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        fk.fk_gauss_sum(X, C, 2.0, w=wt, G=G, logG=logG)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    clocks.stop()
    fk.fk_sync()
    ms = e0.elapsed_time(e1) / steps
    peaks, peak_kind = load_peaks()
    flops = 2.0 * N * K * D
    tflops = flops / (ms * 1e-3) / 1e12
    # one ex2 per (point, centroid) on the special-function units: 16 per SM
    # per clock (4 per sub-partition), the bound this epilogue meets first
    props = torch.cuda.get_device_properties(dev)
    ex2_peak = props.multi_processor_count * SFU_EX2_PER_SM_CLK * SM_MAX_GHZ  # G ex2/s
    ex2_rate = N * K / (ms * 1e-3) / 1e9
    return {"value": round(1e3 / ms, 3), "unit": "calls/s", "ms_per_step": round(ms, 5), "steps": steps,
            "config": {"workload": "gauss_f16", "N": N, "D": D, "K": K, "dtype": "f16", "beta": 2.0,
                       "weights": "uniform in [0.5, 1.5)",
                       "step": "fk_gauss_sum: Gauss-sum bias prep + tensor-core pass with a log-sum-exp epilogue"},
            "roofline": {"bound": "sfu", "kernel": "assign_tc_kernel (Gauss-sum epilogue)",
                         "achieved": round(ex2_rate, 1), "peak": round(ex2_peak, 1), "unit": "G ex2/s",
                         "frac": round(ex2_rate / ex2_peak, 4),
                         "peak_kind": f"ex2: {props.multi_processor_count} SMs x {SFU_EX2_PER_SM_CLK} per clock x "
                                      f"{SM_MAX_GHZ} GHz (derived from unit counts and clock)",
                         "tensor_tflops": round(tflops, 2), "tensor_frac": round(tflops / peaks["bf16_tflops"], 4),
                         "traffic": None},
            "clocks": clocks.summary(w0, w1)}


def measure_fused(args, fk, dev, reps: int):
    """The tiny workload's configured run (5 Lloyd iterations from the first
    K rows) through fk_lloyd_fused: one cooperative launch, X read once per
    iteration.  Timed as `reps` whole runs after 3 untimed ones; the value is
    iterations per second, comparable with the two-stage tiny_f32 line."""
    import torch
    s, w = build_inputs("tiny_f32", dev, 0)
    X = w.X
    N, D, K, iters = s.N, s.D, s.K, s.iters
    C = w.C0.clone()
    labels = torch.empty(N, dtype=torch.int32, device=dev)
    counts = torch.empty(K, dtype=torch.int32, device=dev)
    for _ in range(3):
        C.copy_(w.C0)
        fk.fk_lloyd(X, C, iters, labels=labels, counts=counts, fused=True)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(reps):
        C.copy_(w.C0)
        fk.fk_lloyd(X, C, iters, labels=labels, counts=counts, fused=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    clocks.stop()
    ms = e0.elapsed_time(e1) / (reps * iters)
    props = torch.cuda.get_device_properties(dev)
    fp32_peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * SM_MAX_GHZ / 1e3
    flops = 3.0 * N * K * D  # direct difference: a subtraction and a fused multiply-add per term
    tflops = flops / (ms * 1e-3) / 1e12
    return {"value": round(1e3 / ms, 3), "unit": UNIT, "ms_per_step": round(ms, 5), "steps": reps * iters,
            "config": {"workload": "tiny_f32", "N": N, "D": D, "K": K, "dtype": "f32", "iterations": iters,
                       "step": "fk_lloyd_fused: assignment, exact near-tie re-decision and per-CTA partial sums "
                               "in one pass over X, grid barrier, combine; all iterations in one launch"},
            "roofline": {"bound": "alu", "kernel": "lloyd_fused_kernel", "achieved": round(tflops, 3),
                         "peak": round(fp32_peak, 1), "unit": "TFLOP/s", "frac": round(tflops / fp32_peak, 4),
                         "peak_kind": "fp32 FMA, derived from unit counts and clock",
                         "algorithmic_flops_per_iteration": flops, "traffic": None},
            "clocks": clocks.summary(w0, w1)}


def measure_top2(args, fk, dev, steps: int, warmup: int):
    """The two nearest centroids of the embedding workload's points among its
    K = 1,024 initial centroids (fk_assign_top2: the assignment stage twice,
    the second pass leaving each point's nearest centroid out)."""
    import torch
    s, w = build_inputs("embed_f16", dev, 0)
    X, C = w.X, w.C0.to(torch.float16)
    N, D, K = s.N, s.D, s.K
    l1 = torch.empty(N, dtype=torch.int32, device=dev)
    l2 = torch.empty(N, dtype=torch.int32, device=dev)
    for _ in range(warmup):
        fk.fk_assign_top2(X, C, l1, l2)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        fk.fk_assign_top2(X, C, l1, l2)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    clocks.stop()
    fk.fk_sync()
    ms = e0.elapsed_time(e1) / steps
    peaks, peak_kind = load_peaks()
    flops = 2 * 2.0 * N * K * D  # two assignment passes
    tflops = flops / (ms * 1e-3) / 1e12
    return {"value": round(1e3 / ms, 3), "unit": "calls/s", "ms_per_step": round(ms, 5), "steps": steps,
            "config": {"workload": "top2_f16", "N": N, "D": D, "K": K, "dtype": "f16",
                       "step": "fk_assign_top2: bias prep, two tensor-core assignment passes (the second "
                               "masking each point's nearest centroid), exact re-decision of near-ties after each"},
            "roofline": {"bound": "tensor", "kernel": "assign_tc_kernel (argmin, then argmin with a mask)",
                         "achieved": round(tflops, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tflops / peaks["bf16_tflops"], 4),
                         "peak_kind": f"{peak_kind} bf16 burst (fp16 = bf16 dense rate)",
                         "algorithmic_flops_per_call": flops, "traffic": None},
            "clocks": clocks.summary(w0, w1)}


def measure_seed(args, fk, dev, K: int):
    """k-means++ seeding of the embedding workload (N = 2^20, D = 128, fp16)
    with K centres: one kernel per centre (fp32-screened D2 update reading X
    and D2 once, block weight sums, draw in the last block), plus the first
    round's extra draw kernel.  Timed once after a short warm-up run."""
    import numpy as np
    import torch
    s, w = build_inputs("embed_f16", dev, 0)
    u = np.random.default_rng(7).random(K)
    fk.fk_seed_kmeanspp(w.X, 8, u[:8])
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    fk.fk_seed_kmeanspp(w.X, K, u)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    peaks, peak_kind = load_peaks()
    bytes_per_round = s.N * s.D * 2 + s.N * 8  # X and D2 read (D2 is written only where it drops)
    gbs = (K - 1) * bytes_per_round / (ms * 1e-3) / 1e9
    return {"value": round(1e3 / ms, 4), "unit": "seedings/s", "ms_per_step": round(ms, 3), "steps": 1,
            "config": {"workload": "seed_f16", "N": s.N, "D": s.D, "K": K, "dtype": "f16",
                       "step": "fk_seed_kmeanspp: K - 1 rounds of D2 update + draw"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": f"{peak_kind} copy",
                         "algorithmic_bytes_per_round": bytes_per_round, "traffic": None}}


OTHER_WORKLOADS = ("tiny_f32", "tiny_f32_fused", "batched_bf16", "zipf_bf16", "embed_f32", "gauss_f16", "top2_f16",
                   "seed_f16", "ooc_f16")


def bench_gpu(args):
    import torch

    import distance_argmin_flashassign_b200 as fk
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    head, s, w = measure(args, args.workload, fk, dev, world, rank, args.steps, args.warmup,
                         args.cpu_budget if args.cpu else 0.0, seed=rank)
    out = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": s.dtype, "data": "synthetic",
           "config": dict(head["config"], parallelism="replicas" if world > 1 else "single GPU"),
           "roofline": head["roofline"], "roofline_update": head["roofline_update"],
           "gpu_launches": head["gpu_launches"], "clocks": head["clocks"]}
    if args.e2e:
        out["e2e"] = bench_e2e(args, s, w, fk, dev, world)
    if "cpu_baseline" in head:
        out["cpu_baseline"] = head["cpu_baseline"]
    del w
    torch.cuda.empty_cache()
    # the other configured workloads, each measured the same way (one GPU)
    if args.all_workloads and world == 1:
        others = {}
        pick = set(args.others.split(",")) - {""}
        unknown = pick - set(OTHER_WORKLOADS)
        if unknown:
            raise SystemExit(f"unknown workloads in --others: {sorted(unknown)}")
        for name in [n for n in ("tiny_f32", "batched_bf16", "zipf_bf16", "embed_f32") if n != args.workload and n in pick]:
            steps = args.steps if name not in ("zipf_bf16", "embed_f32") else max(3, min(args.steps, 20 if name == "embed_f32" else 5))
            res, _, wk = measure(args, name, fk, dev, world, rank, steps, max(3, min(args.warmup, 5)),
                                 args.other_cpu_budget if args.cpu else 0.0, seed=rank)
            others[name] = res
            del wk
            torch.cuda.empty_cache()
        if "tiny_f32_fused" in pick:
            others["tiny_f32_fused"] = measure_fused(args, fk, dev, max(3, min(args.steps, 40)))
        if "gauss_f16" in pick:
            others["gauss_f16"] = measure_gauss(args, fk, dev, max(3, min(args.steps, 50)), 3)
        if "top2_f16" in pick:
            others["top2_f16"] = measure_top2(args, fk, dev, max(3, min(args.steps, 50)), 3)
        if "seed_f16" in pick:
            others["seed_f16"] = measure_seed(args, fk, dev, 1024)
        torch.cuda.empty_cache()
        if args.ooc_rows_all > 0 and "ooc_f16" in pick:
            others["ooc_f16"] = run_ooc(args, fk, dev, args.ooc_rows_all,
                                        args.other_cpu_budget if args.cpu else 0.0)
        out["workloads"] = others
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def bench_e2e(args, s, w, fk, dev, world):
    """Same metric through fk_lloyd_ooc with host buffers: every step copies X
    (pinned) to the device in chunks, runs one Lloyd iteration and copies the
    labels, centroids and counts back."""
    import torch
    B, N, D, K = s.B, s.N, s.D, s.K
    if B != 1:
        return None
    Xh = w.X.cpu().pin_memory()
    Ch = w.C0.cpu().clone()
    lab_h = torch.empty(N, dtype=torch.int32).pin_memory()
    cnt_h = torch.empty(K, dtype=torch.int32).pin_memory()
    chunk = max(1, N // 4)
    stream = torch.cuda.current_stream(dev)
    for _ in range(min(args.warmup, 2)):
        fk.fk_lloyd_ooc(Xh, Ch, 1, chunk, lab_h, cnt_h)
    steps = max(1, min(args.steps, args.e2e_steps))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(steps):
        fk.fk_lloyd_ooc(Xh, Ch, 1, chunk, lab_h, cnt_h)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    value, _ = aggregate(steps, t0.elapsed_time(t1), world, dev)
    es = s.bytes_per_elem
    return {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": N * D * es + K * D * 4,
            "d2h_bytes_per_step": N * 4 + K * D * 4 + K * 4, "steps": steps,
            "api": "fk_lloyd_ooc(iters=1, chunk_rows=N/4), pinned host X"}


# ---------------------------------------------------------- out of core --
def ooc_inputs(rows: int, device):
    """X of the out-of-core workload with ``rows`` rows in pinned host memory
    (generated on the device block by block, same recipe as the full
    workload's first rows), and its configured initial centroids."""
    import torch

    import workloads
    s = workloads.spec("ooc_f16", N=rows)
    Xh = torch.empty((rows, s.D), dtype=torch.float16, pin_memory=True)
    cen = workloads.centers(s, 0, device)
    piece = 1 << 24
    for r0 in range(0, rows, piece):
        Xh[r0:r0 + piece].copy_(workloads.rows(s, r0, min(rows, r0 + piece), device=device, cen=cen))
    return s, Xh, Xh[: s.K].float().clone()  # init = first K rows


def run_ooc(args, fk, dev, rows: int, cpu_budget: float):
    """The configured iterations of the out-of-core workload (at `rows` rows)
    in one fk_lloyd_ooc call: every chunk of X crosses the host link once per
    iteration on a copy stream while the previous chunk is assigned and
    accumulated.  The host-to-device rate is reported against a plain copy
    of one chunk from the same pinned buffer, timed in this process."""
    import torch
    s, Xh, C0 = ooc_inputs(rows, dev)
    N, D, K, chunk, iters = s.N, s.D, s.K, s.chunk_rows, s.iters
    stream = torch.cuda.current_stream(dev)
    # the plain pinned-to-device copy rate of one chunk
    dchunk = torch.empty((min(chunk, N), D), dtype=torch.float16, device=dev)
    dchunk.copy_(Xh[: dchunk.shape[0]], non_blocking=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        dchunk.copy_(Xh[: dchunk.shape[0]], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    copy_gbs = 3 * dchunk.numel() * 2 / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del dchunk
    torch.cuda.empty_cache()

    lab_h = torch.empty(N, dtype=torch.int32, pin_memory=True)
    cnt_h = torch.empty(K, dtype=torch.int32)
    Ch = C0.clone()
    fk.fk_lloyd_ooc(Xh, Ch, 1, chunk, lab_h, cnt_h)  # warm-up: sets up the device ring and workspace
    torch.cuda.synchronize(dev)
    Ch = C0.clone()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    n0 = fk.fk_launch_count()
    w0 = time.time()
    e0.record(stream)
    fk.fk_lloyd_ooc(Xh, Ch, iters, chunk, lab_h, cnt_h)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    launches = fk.fk_launch_count() - n0
    clocks.stop()
    ms = e0.elapsed_time(e1)
    value = iters / (ms * 1e-3)
    h2d_gbs = iters * N * D * 2 / (ms * 1e-3) / 1e9
    nchunks = (N + chunk - 1) // chunk
    out = {"value": round(value, 4), "unit": UNIT, "ms_per_step": round(ms / iters, 3), "steps": iters,
           "warmup": 1,
           "config": {"workload": "ooc_f16", "N": N, "N_configured": 10 ** 9, "D": D, "K": K, "B": 1,
                      "dtype": s.dtype, "chunk_rows": chunk, "chunks_per_iteration": nchunks,
                      "iterations_configured": iters,
                      "step": "one Lloyd iteration streamed from pinned host memory (fk_lloyd_ooc, "
                              f"{iters} iterations in one call)",
                      "reduced_N": "the configured 10^9 rows need 256 GB of pinned host memory"},
           "roofline": {"bound": "host-to-device copy", "achieved": round(h2d_gbs, 2),
                        "peak": round(copy_gbs, 2), "unit": "GB/s", "frac": round(h2d_gbs / copy_gbs, 4),
                        "peak_kind": "plain copy of one chunk from the same pinned buffer, measured in this run",
                        "traffic": None},
           "gpu_launches": launches, "clocks": clocks.summary(w0, w1),
           "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": N * D * 2 + K * D * 4,
                   "d2h_bytes_per_step": K * D * 4 + K * 4 + (N * 4) // iters}}
    if cpu_budget > 0:
        import workloads
        n = min(N, 1 << 16)
        Xs = workloads.rows(s, 0, n, device=dev).cpu()
        v, n_used, reps, secs, cores = oracle_throughput(Xs.double().numpy(), C0.double().numpy(), s.dtype, N,
                                                         cpu_budget)
        out["cpu_baseline"] = {"value": round(v, 8), "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x {n_used} of {N} rows against all {K} centroids, one Lloyd "
                                         f"step each ({secs:.1f} s in all), scaled linearly in N"}
    del Xh, lab_h
    return out


def bench_ooc(args):
    import torch

    import distance_argmin_flashassign_b200 as fk
    rank, world, local = dist_env()
    if world > 1:
        raise SystemExit("ooc_f16 runs on one GPU (its pinned host copy of X does not fit once per rank)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    r = run_ooc(args, fk, dev, args.ooc_rows, args.cpu_budget if args.cpu else 0.0)
    out = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": 1, "steps": r["steps"], "warmup": 1,
           "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f16", "data": "synthetic"}
    out.update({k: v for k, v in r.items() if k not in ("value", "unit", "ms_per_step", "steps", "warmup")})
    print(json.dumps(out), flush=True)


# -------------------------------------------------------- reference arm --
def bench_reference(args):
    """The oracle, as it stands, on the host cores: each step is one Lloyd
    step of the oracle on a bounded row sample of the same workload, scaled
    linearly in N.  Only rank 0 works and prints under torchrun."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch

    import workloads
    s = workloads.spec(args.workload)
    per_step = max(0.05, args.ref_budget / max(1, args.steps + args.warmup))
    if s.name == "ooc_f16":  # the same reduced N as the own arm; a row sample only
        s = s.replace(N=args.ooc_rows)
        X64 = workloads.rows(s, 0, min(s.N, 1 << 16)).double().numpy()
        C64 = X64[: s.K].copy()
    else:
        w = workloads.make(s.replace(B=1) if s.B > 1 else s, seed=0, device="cpu")
        X64 = w.X.double().numpy()
        C64 = w.C0.double().numpy()
    import oracle
    lib = oracle.load()
    t = time.perf_counter()
    oracle.lloyd_step(X64[:128], C64, s.dtype, lib)
    per_row = (time.perf_counter() - t) / 128
    n = int(max(64, min(X64.shape[0], per_step / max(per_row, 1e-9))))
    for _ in range(args.warmup):
        oracle.lloyd_step(X64[:n], C64, s.dtype, lib)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.lloyd_step(X64[:n], C64, s.dtype, lib)
    dt = time.perf_counter() - t
    value = args.steps * n / (s.N * s.B * dt)
    out = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(1e3 / value, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": args.workload, "N": s.N, "D": s.D, "K": s.K, "B": s.B, "dtype": s.dtype,
                      "step": "one Lloyd iteration of the fp64 CPU oracle on a row sample"},
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "kind": "oracle",
                            "cores": oracle.num_threads(),
                            "sample": f"{n} of {s.N * s.B} rows per step against all {s.K} centroids, "
                                      f"scaled linearly in N"},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    del torch


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default="embed_f16")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu", dest="cpu", action="store_false")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds of oracle work for --impl reference")
    ap.add_argument("--no-all", dest="all_workloads", action="store_false",
                    help="measure the headline workload only (skip the other configured workloads)")
    ap.add_argument("--rows", type=int, default=0,
                    help="rows per problem of the headline workload (0: as configured); for profiling smaller cases")
    ap.add_argument("--others", default=",".join(OTHER_WORKLOADS),
                    help="comma-separated subset of the other workloads to measure after the headline one")
    ap.add_argument("--other-cpu-budget", type=float, default=5.0,
                    help="seconds of oracle work for each other workload's cpu_baseline")
    ap.add_argument("--ooc-rows-all", type=int, default=1 << 27,
                    help="rows of the out-of-core workload in the default line (2^27: 32 GiB pinned, 2 chunks; "
                         "0 skips it)")
    ap.add_argument("--ooc-rows", type=int, default=1 << 28,
                    help="rows of the out-of-core workload (default 2^28: 64 GiB of pinned fp16, 4 chunks)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps, reported as run
    if args.impl == "reference":
        bench_reference(args)
    elif args.workload == "ooc_f16":
        bench_ooc(args)
    else:
        bench_gpu(args)


if __name__ == "__main__":
    main()
