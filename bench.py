#!/usr/bin/env python
"""Benchmark of the causal sequence convolution on B200.

One step = one call of the fused causal convolution (load, pad, FFT, spectral
product, inverse FFT, truncate, store) over one batch of the named workload
(default: the Caracal-Small-shaped fp32 MHF convolution, B=8, L=1024, D=768).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

For N > 1 launch under torchrun: every rank convolves its own batch (its own
seed) on its own GPU with no collective on the data path (weak scaling);
timing is the max over ranks.  Prints one JSON line on rank 0.

Timing: inputs larger than L2 -- the step rotates through enough copies of
(v, g, r) that each step touches buffers last used more than 126 MB of traffic
ago; CUDA events on the launching stream bracket the K timed steps, with a
barrier and a device synchronize on both sides.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "causal FFT-conv GB/s and (B*D*L)/s at 1 B200; % of HBM roofline"
L2_BYTES = 126 * 2 ** 20
# the device code each kernel is built from (api.cu holds host code and table storage)
_FUSED_SOURCES = ["fftconv_fused.cuh", "fft_reg.cuh", "tma.cuh", "configs_fused.cuh"]
KERNEL_SOURCES = {
    "fftconv_fused_kernel": _FUSED_SOURCES,
    "bigrow_group_kernel": ["bigconv.cuh", "configs_rows.cuh"] + _FUSED_SOURCES,
    "bigconv_kernel": ["bigconv.cuh", "configs_rows.cuh"] + _FUSED_SOURCES,
    "hr_mid_kernel": ["hbmrows.cuh"] + _FUSED_SOURCES,
    "ntt_conv_kernel": ["ntt.cuh"],
    "tcconv_kernel": ["tcconv.cuh", "tcgen05.cuh", "tma.cuh"],
    "mhf_gate_kernel": ["mhf_gate.cuh", "tcgen05.cuh", "tma.cuh"],
    "dwconv_vec_kernel": ["dwconv.cuh"],
}
DWCONV_METRIC = "causal depthwise conv GB/s (x in, y out) at 1 B200; % of HBM roofline"
GATE_METRIC = "MHF gate stream + causal FFT-conv GB/s (v, a in, r out) at 1 B200; % of HBM roofline"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="small_f32",
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.GATE_WORKLOADS)
                    + sorted(workloads.DWCONV_WORKLOADS),
                    help="a convolution workload, a gate workload (MHF gate stream + convolution) "
                         "or a depthwise-convolution workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--path", choices=["fwd", "bwd", "decode"], default="fwd",
                    help="fwd: the causal convolution (default line); bwd: its gradients (dv, dg); "
                         "decode: one autoregressive step at t = L-1 from [B, L, D] caches")
    ap.add_argument("--shape", default=None,
                    help="B,L,D override of the workload's sizes (same recipe); for small profiler captures")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config list (the other convolution workloads timed in the same run)")
    ap.add_argument("--per-config-steps", type=int, default=200,
                    help="timed steps of each per_config entry (graph-replayed)")
    ap.add_argument("--probe", action="store_true",
                    help="measure the per-SM rates behind the ALU rooflines (FFMA, FFMA2, IMAD, IMAD.HI, "
                         "shared memory, distributed shared memory) and print them as one JSON line")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_seed(w: workloads.Workload, rank: int) -> int:
    """Each rank convolves its own batch: the workload's seed for rank 0, a
    distinct one for the others (weak scaling, no data shared across ranks)."""
    return w.seed + 1000 * rank


def max_over_ranks(value: float, pg, device=None) -> float:
    """Max of a per-rank timing over the process group (identity without one)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank: int, world: int, steps: int, ms: float, bytes_per_unit: int):
    """Whole-job outputs/s and algorithmic GB/s from the max-over-ranks time."""
    units = units_per_rank * world * steps
    return units / (ms * 1e-3), units * bytes_per_unit / (ms * 1e-3) / 1e9


def _code_only(text: str) -> str:
    """C++ source without comments and whitespace (edits to comments do not
    change the code a kernel is compiled from)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def kernel_source_hash(kernel: str) -> str:
    """sha256 (16 hex digits) of the device code `kernel` is built from: its
    sources with comments and whitespace removed."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        p = os.path.join(ROOT, "spectral_sequence_mixing_b200", "csrc", f)
        if os.path.exists(p):
            h.update(_code_only(open(p).read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_counters(workload: str, kernel: str):
    """(DRAM bytes read + write, ALU lane operations, their pipe "fp32" or
    "imad") per launch of `kernel` on the full-size `workload`, from
    profiles/kernel_counters.txt (lines: workload kernel source_hash
    dram_bytes alu_lane_ops pipe), if they were taken on the current kernel
    sources; else (None, None, None)."""
    p = os.path.join(ROOT, "profiles", "kernel_counters.txt")
    if not os.path.exists(p):
        return None, None, None
    kernel = kernel.split(" (")[0]  # "hr_mid_kernel (four-step: ...)" -> the kernel name
    for line in open(p):
        f = line.split()
        if len(f) == 6 and not line.startswith("#") and f[0] == workload and f[1] == kernel:
            if f[2] != kernel_source_hash(kernel):
                return None, None, None
            return float(f[3]), float(f[4]), f[5]
    return None, None, None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    @staticmethod
    def _handle(pynvml, index: int):
        """NVML handle of CUDA device `index`, found by PCI address (CUDA and
        NVML may number devices differently); by index if that fails."""
        try:
            import torch
            pr = torch.cuda.get_device_properties(index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(index)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def report(self):
        if self._nv is None:
            return None
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def cpu_oracle_rate(w: workloads.Workload, v, g, budget_s: float):
    """Time the oracle on whole rows of the workload: channel slices [B, L, k]
    with k doubling until about budget_s of CPU work.  Returns (units/s,
    threads, description, seconds)."""
    import oracle
    fv = workloads.bf16_to_f32(v) if w.dtype == "bf16" else v
    fg = workloads.bf16_to_f32(g) if w.dtype == "bf16" else g
    k, spent, units, secs = 1, 0.0, 0, 0.0
    while True:
        k = min(k, w.D)
        sv = np.ascontiguousarray(fv[:, :, :k])
        sg = np.ascontiguousarray(fg[:, :, :k])
        t0 = time.perf_counter()
        if w.dtype == "i32":
            oracle.causal_conv_int(sv, sg)
        else:
            oracle.causal_conv(sv, sg)
        dt = time.perf_counter() - t0
        units, secs = w.B * w.L * k, dt
        spent += dt
        if spent >= budget_s / 3 or k == w.D or dt * 2 > budget_s - spent:
            break
        k *= 2
    reps = 1
    if k == w.D and secs < budget_s / 3:
        # the whole workload is cheap: repeat it to time about budget_s of work
        reps = max(1, min(64, int(budget_s / max(secs, 1e-3))))
        t0 = time.perf_counter()
        for _ in range(reps):
            if w.dtype == "i32":
                oracle.causal_conv_int(sv, sg)
            else:
                oracle.causal_conv(sv, sg)
        units, secs = w.B * w.L * k * reps, time.perf_counter() - t0
    desc = (f"oracle on channels [0,{k}) of {w.name}: {w.B}x{w.L}x{k} outputs (whole rows)"
            + (f", {reps} passes" if reps > 1 else ""))
    return units / secs, oracle.num_threads(), desc, secs


def workload_for(args) -> workloads.Workload:
    w = workloads.WORKLOADS[args.workload]
    if args.shape:
        B, L, D = (int(x) for x in args.shape.split(","))
        from dataclasses import replace
        w = replace(w, B=B, L=L, D=D)
    return w


def run_reference(args, rank, world):
    """The oracle (plain CPU direct sum) timed on the host cores as the
    reference arm, on the same workload and metric."""
    if rank != 0:
        return
    w = workload_for(args)
    v, g = workloads.generate(w, B=w.B, L=w.L, D=w.D)
    per_step = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    import oracle
    fv = workloads.bf16_to_f32(v) if w.dtype == "bf16" else v
    fg = workloads.bf16_to_f32(g) if w.dtype == "bf16" else g
    # calibrate the channel count k per step against the per-step budget
    k = 1
    while True:
        t0 = time.perf_counter()
        sv, sg = np.ascontiguousarray(fv[:, :, :k]), np.ascontiguousarray(fg[:, :, :k])
        (oracle.causal_conv_int if w.dtype == "i32" else oracle.causal_conv)(sv, sg)
        dt = time.perf_counter() - t0
        if dt * 2 > per_step or k >= w.D:
            break
        k = min(w.D, k * 2)
    sv, sg = np.ascontiguousarray(fv[:, :, :k]), np.ascontiguousarray(fg[:, :, :k])
    fn = oracle.causal_conv_int if w.dtype == "i32" else oracle.causal_conv
    for _ in range(args.warmup):
        fn(sv, sg)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn(sv, sg)
    el = time.perf_counter() - t0
    units = w.B * w.L * k * args.steps
    gbs = units * 3 * w.elem_bytes / el / 1e9
    sample = f"oracle on channels [0,{k}) of {w.name} per step ({w.B}x{w.L}x{k} outputs, whole rows)"
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"f32": "f64", "bf16": "f64", "i32": "int64"}[w.dtype], "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "L": w.L, "D": w.D, "io_dtype": w.dtype},
        "outputs_per_s": units / el,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def dominant_kernel(w: workloads.Workload, four_step: bool) -> str:
    """The kernel that does a forward call's transform on workload `w`."""
    if w.dtype == "i32":
        return "ntt_conv_kernel"
    if w.L <= 1024:
        return "fftconv_fused_kernel"
    if w.L <= 2048:
        return "bigrow_group_kernel"
    if w.L <= 4096:
        return "tcconv_kernel" if w.dtype == "bf16" else "bigrow_group_kernel"
    return ("hr_mid_kernel (four-step path: the norm, alpha, fwd, mid and inv launches of a step; traffic and "
            "ALU counts are the whole step's)") if four_step else "bigconv_kernel"


def probe_rates():
    """Measured lane operations per clock per SM of each pipe, from
    profiles/probe_rates.txt (written from a `bench.py --probe` run), or {}."""
    p = os.path.join(ROOT, "profiles", "probe_rates.txt")
    rates = {}
    if os.path.exists(p):
        for line in open(p):
            f = line.split()
            if len(f) == 2 and not line.startswith("#"):
                rates[f[0]] = float(f[1])
    return rates


def alu_roofline(alu_ops, alu_pipe, ms_per_step, clocks):
    """Executed lane operations of the kernel's busiest ALU pipe (ncu, same
    sources) per launch against 148 SMs x the measured lanes/clk of that pipe
    (bench.py --probe; nominal FP32 128, IMAD 64 when no probe is recorded) x
    the SM clock sampled during the run."""
    measured = probe_rates().get(alu_pipe)
    lanes = measured if measured else {"fp32": 128, "imad": 64}[alu_pipe]
    sm_hz = clocks["sm_mhz"] * 1e6 if clocks and clocks.get("sm_mhz") else 1.965e9
    peak = 148 * lanes * sm_hz / 1e9
    achieved = alu_ops / (ms_per_step * 1e-3) / 1e9
    src = (f"148 SMs x {lanes:g} lanes/clk measured by bench.py --probe x sampled SM clock" if measured
           else f"148 SMs x {lanes} lanes/clk (nominal) x sampled SM clock")
    return {"bound": "alu", "pipe": alu_pipe, "achieved": achieved, "peak": peak,
            "unit": f"G {alu_pipe.upper()} lane-op/s", "frac": achieved / peak, "lane_ops_per_launch": alu_ops,
            "peak_source": src}


def time_config(w: workloads.Workload, rank, world, dev, pg, steps: int, warmup: int, cpu_budget_s: float):
    """One forward workload timed in this run: rotating buffer sets larger than
    L2 (cold L2), the steps replayed from CUDA graphs (a step is one library
    call, 1 or 4 launches), CUDA events on the replay stream, max over ranks;
    plus the same steps on one set (hot L2) and a short oracle sample."""
    import torch
    import spectral_sequence_mixing_b200 as ssm
    v_np, g_np = workloads.generate(w, seed=rank_seed(w, rank))
    if w.dtype == "bf16":
        hv = torch.from_numpy(v_np.view(np.int16)).view(torch.bfloat16)
        hg = torch.from_numpy(g_np.view(np.int16)).view(torch.bfloat16)
    else:
        hv, hg = torch.from_numpy(v_np), torch.from_numpy(g_np)
    v0, g0 = hv.to(dev), hg.to(dev)
    set_bytes = 3 * w.units * w.elem_bytes
    n_sets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    sets = [(v0, g0, torch.empty_like(v0))] + [(v0.clone(), g0.clone(), torch.empty_like(v0))
                                                for _ in range(n_sets - 1)]
    n_ws = ssm.fast_workspace_bytes(v0.dtype, w.B, w.L, w.D)
    ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)

    def step(i):
        a, b, c = sets[i % n_sets]
        ssm.causal_conv(a, b, out=c, workspace=ws)  # on the current (capture) stream

    G = n_sets * max(1, 32 // n_sets)
    with torch.cuda.stream(side):
        for i in range(max(3, warmup)):
            step(i)
        side.synchronize()
        cold = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cold, stream=side):
            for i in range(G):
                step(i)
        hot = torch.cuda.CUDAGraph()
        with torch.cuda.graph(hot, stream=side):
            for i in range(G):
                step(0)
    torch.cuda.synchronize(dev)
    reps = max(1, math.ceil(steps / G))

    def timed(graph):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(side):
            graph.replay()  # warm replay
            if pg is not None:
                pg.barrier()
            torch.cuda.synchronize(dev)
            e0.record(side)
            for _ in range(reps):
                graph.replay()
            e1.record(side)
            torch.cuda.synchronize(dev)
            if pg is not None:
                pg.barrier()
        return max_over_ranks(e0.elapsed_time(e1), pg, dev) / (reps * G)

    with ClockSampler(dev.index) as clk:
        ms = timed(cold)
    ms_hot = timed(hot)
    clocks = clk.report()
    del cold, hot
    alg = w.algorithmic_bytes
    peak, peak_src = measured_peaks()
    kernel = dominant_kernel(w, n_ws > 0)
    achieved = alg / (ms * 1e-3) / 1e9
    traffic, alu_ops, alu_pipe = recorded_counters(w.name, kernel)
    entry = {
        "workload": w.name, "B": w.B, "L": w.L, "D": w.D, "io_dtype": w.dtype,
        "transform_len": 2 ** math.ceil(math.log2(2 * w.L)),
        "ms_per_step": ms, "steps": reps * G, "value": achieved * world, "unit": "GB/s",
        "outputs_per_s": w.units * world / (ms * 1e-3),
        "launch": f"CUDA graph replay of {G} steps ({5 if n_ws else 1} launches per step)",
        "l2": f"cold: {n_sets} rotating (v,g,r) sets of {set_bytes / 2 ** 20:.1f} MiB",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "kernel": kernel,
                     "algorithmic_bytes_per_launch": alg, "traffic": traffic},
        "hot_l2": {"ms_per_step": ms_hot, "GB/s": alg / (ms_hot * 1e-3) / 1e9,
                   "note": "the same steps on one (v,g,r) set"},
        "clocks": clocks,
    }
    if alu_ops:
        entry["alu_roofline"] = alu_roofline(alu_ops, alu_pipe, ms, clocks)
    if rank == 0 and world == 1 and cpu_budget_s > 0:
        cpu_ups, cores, desc, secs = cpu_oracle_rate(w, v_np, g_np, budget_s=cpu_budget_s)
        entry["cpu_baseline"] = {"value": cpu_ups * 3 * w.elem_bytes / 1e9, "unit": "GB/s", "cores": cores,
                                 "kind": "oracle", "sample": desc, "seconds": secs}
    del sets, ws, v0, g0
    torch.cuda.empty_cache()
    return entry


def run_ours(args, rank, world, local):
    import torch
    import spectral_sequence_mixing_b200 as ssm

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    w = workload_for(args)
    v_np, g_np = workloads.generate(w, seed=rank_seed(w, rank))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "i32": torch.int32}[w.dtype]

    def to_t(x):
        if w.dtype == "bf16":
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(x)

    hv, hg = to_t(v_np), to_t(g_np)
    v0, g0 = hv.to(dev), hg.to(dev)
    set_bytes = 3 * w.units * w.elem_bytes
    n_sets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    sets = [(v0, g0, torch.empty_like(v0))] + [(v0.clone(), g0.clone(), torch.empty_like(v0)) for _ in
                                                range(n_sets - 1)]
    stream = torch.cuda.current_stream(dev)
    # optional workspace of the four-step long-row path: norm partials, row
    # scales, the forward pass, the middle pass and the inverse pass per conv
    n_ws = ssm.fast_workspace_bytes(tdt, w.B, w.L, w.D)
    ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
    conv_launches = 5 if n_ws else 1
    if args.path == "fwd":
        def fn(a, b, out, stream):
            ssm.causal_conv(a, b, out=out, workspace=ws, stream=stream)
        bytes_per_step, launches_per_step = 3 * w.units * w.elem_bytes, conv_launches
    elif args.path == "bwd":
        # dr is the third buffer of the set; dv, dg get their own buffers
        bwd_out = [(torch.empty_like(v0), torch.empty_like(v0)) for _ in range(n_sets)]

        def fn(a, b, out, stream, _k=[0]):
            dv, dg = bwd_out[_k[0] % n_sets]
            _k[0] += 1
            ssm.causal_conv_bwd(out, a, b, dv=dv, dg=dg, workspace=ws, stream=stream)
        for _, _, c in sets:
            c.copy_(sets[0][0])
        bytes_per_step, launches_per_step = 5 * w.units * w.elem_bytes, 2 * conv_launches
    else:
        dec_ws = torch.empty(ssm.decode_workspace_bytes(v0.dtype, w.B, w.D, w.L - 1), dtype=torch.uint8, device=dev)
        dec_out = torch.empty((w.B, w.D), dtype=v0.dtype, device=dev)

        def fn(a, b, out, stream):
            ssm.causal_conv_decode(a, b, w.L - 1, out=dec_out, workspace=dec_ws, stream=stream)
        bytes_per_step, launches_per_step = (2 * w.L + 1) * w.B * w.D * w.elem_bytes, 2

    for i in range(args.warmup):
        a, b, c = sets[i % n_sets]
        fn(a, b, out=c, stream=stream)
    torch.cuda.synchronize(dev)

    # The timed steps are replayed from CUDA graphs of the same library calls
    # (one graph of G consecutive steps, whole rotations of the buffer sets,
    # and one graph per set for the remainder), so exactly K steps run with
    # no host launch gaps between them.
    side = torch.cuda.Stream(dev)
    # one graph holds the whole timed region when it is short (one host launch)
    G = args.steps if args.steps <= 256 else n_sets * max(1, 32 // n_sets)
    with torch.cuda.stream(side):
        big = torch.cuda.CUDAGraph()
        with torch.cuda.graph(big, stream=side):
            for i in range(G):
                a, b, c = sets[i % n_sets]
                fn(a, b, out=c, stream=side)
        singles = []
        for k in range(n_sets):
            gk = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gk, stream=side):
                a, b, c = sets[k]
                fn(a, b, out=c, stream=side)
            singles.append(gk)
    torch.cuda.synchronize(dev)

    def run_steps(n):
        for _ in range(n // G):
            big.replay()
        for i in range(n % G):
            singles[i % n_sets].replay()

    with torch.cuda.stream(side):
        run_steps(max(G, args.warmup))  # warm replays of the captured graphs
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(side):
            start.record(side)
            run_steps(args.steps)
            end.record(side)
        torch.cuda.synchronize(dev)
        barrier()
    del big, singles
    ms = max_over_ranks(start.elapsed_time(end), pg, dev)
    ms_per_step = ms / args.steps
    units_step = w.units if args.path != "decode" else w.B * w.D
    ups, _ = throughput(units_step, world, args.steps, ms, 1)
    gbs = bytes_per_step * world * args.steps / (ms * 1e-3) / 1e9

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    phv, phg = hv.pin_memory(), hg.pin_memory()
    phr = torch.empty_like(phv).pin_memory()
    dv, dg, dr = sets[0]
    for _ in range(2):
        ssm.causal_conv_from_host(phv, phg, phr, dv, dg, dr, workspace=ws, stream=stream)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        ssm.causal_conv_from_host(phv, phg, phr, dv, dg, dr, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    _, e2e_gbs = throughput(w.units, world, e2e_steps, ems, 3 * w.elem_bytes)

    peak, peak_src = measured_peaks()
    kernel = "decode_partial_kernel" if args.path == "decode" else dominant_kernel(w, n_ws > 0)
    per_launch_bytes = bytes_per_step // 2 if args.path == "bwd" else bytes_per_step
    achieved = bytes_per_step / (ms_per_step * 1e-3) / 1e9
    traffic, alu_ops, alu_pipe = ((None, None, None) if (args.shape or args.path != "fwd")
                                  else recorded_counters(w.name, kernel))
    clocks = clk.report()
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"f32": "f32", "bf16": "f32", "i32": "u32"}[w.dtype], "data": "synthetic",
        "config": {"workload": w.name, "path": args.path, "B": w.B, "L": w.L, "D": w.D, "io_dtype": w.dtype,
                   "transform_len": 2 ** math.ceil(math.log2(2 * w.L)),
                   "l2": f"inputs larger than L2: {n_sets} rotating (v,g,r) sets of {set_bytes / 2 ** 20:.0f} MiB",
                   "launch": f"timed steps replayed from CUDA graphs ({G} steps per graph)",
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "outputs_per_s": ups,
        "hbm_frac": gbs / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                     "kernel": kernel, "algorithmic_bytes_per_launch": per_launch_bytes, "traffic": traffic},
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": 2 * w.units * w.elem_bytes,
                "d2h_bytes_per_step": w.units * w.elem_bytes, "steps": e2e_steps,
                "path": "causal_conv_from_host (pinned host buffers)"},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
    }
    if alu_ops and launches_per_step == 1:
        # the transform kernels are bound by ALU issue, not by HBM
        line["alu_roofline"] = alu_roofline(alu_ops, alu_pipe, ms_per_step, clocks)
    if args.path != "fwd":  # the host-buffer leg and CPU baseline describe the forward line only
        line.pop("e2e")
        args.no_cpu_baseline = True
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_ups, cores, desc, secs = cpu_oracle_rate(w, v_np, g_np, budget_s=15.0)
        line["cpu_baseline"] = {"value": cpu_ups * 3 * w.elem_bytes / 1e9, "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "sample": desc, "seconds": secs}
    if args.path == "fwd" and not args.shape and not args.no_per_config:
        # every convolution workload on the same clock: the line's own
        # workload again (hot and cold L2, graph-replayed), then the others
        del sets, ws
        torch.cuda.empty_cache()
        order = [w.name] + [n for n in workloads.WORKLOADS if n != w.name]
        line["per_config"] = [
            time_config(workloads.WORKLOADS[n], rank, world, dev, pg, args.per_config_steps, args.warmup,
                        0.0 if n == w.name or args.no_cpu_baseline else 2.5)
            for n in order]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def gate_oracle_rate(gw, v, a, w, bias, budget_s: float):
    """Time the oracle (gate, then convolution) on whole heads of batch 0,
    repeated to about budget_s.  Returns (units/s, threads, description, seconds)."""
    import oracle
    import oracle.mhf_gate as mhf
    C = gw.D // gw.H
    sv, sa = np.ascontiguousarray(v[:1, :, :C]), np.ascontiguousarray(a[:1, :, :C])
    sw, sb = np.ascontiguousarray(w[:C]), np.ascontiguousarray(bias[:C])
    reps, secs = 0, 0.0
    t0 = time.perf_counter()
    while secs < budget_s and reps < 1000:
        mhf.mhf_gated_conv(sv, sa, sw, sb, 1)
        reps += 1
        secs = time.perf_counter() - t0
    units = gw.L * C * reps
    desc = f"oracle (gate + direct sum) on head 0 of batch 0 of {gw.name}: 1x{gw.L}x{C} outputs, {reps} passes"
    return units / secs, oracle.num_threads(), desc, secs


def run_gated(args, rank, world, local):
    """The MHF gate stream + convolution on a gate workload: one step = one
    call of mhf_gated_conv (the tcgen05 gate kernel, then the convolution)."""
    import torch
    import spectral_sequence_mixing_b200 as ssm

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    gw = workloads.GATE_WORKLOADS[args.workload]
    v, a, w, bias = workloads.generate_gate(gw.B, gw.L, gw.D, gw.H, gw.K, gw.dtype, gw.seed + 1000 * rank)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[gw.dtype]
    es = 4 if gw.dtype == "f32" else 2

    def to_t(x):
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if gw.dtype == "bf16" else torch.from_numpy(x)

    hv, ha = to_t(v), to_t(a)
    tw, tb = torch.from_numpy(w).to(dev), torch.from_numpy(bias).to(dev)
    units = gw.units
    set_bytes = 4 * units * es  # v, a, gate workspace, r
    n_sets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    v0, a0 = hv.to(dev), ha.to(dev)
    ws_bytes = ssm.mhf_gated_conv_workspace_bytes(tdt, gw.B, gw.L, gw.D)
    sets = [(v0 if i == 0 else v0.clone(), a0 if i == 0 else a0.clone(),
             torch.empty(ws_bytes, dtype=torch.uint8, device=dev), torch.empty_like(v0)) for i in range(n_sets)]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        sv, sa, sws, sr = sets[i % n_sets]
        ssm.mhf_gated_conv(sv, sa, tw, tb, gw.H, out=sr, workspace=sws, stream=stream)

    def timed(fn, steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(steps):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), pg, dev)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        ms = timed(step, args.steps)
    clocks = clk.report()
    ms_per_step = ms / args.steps
    alg_bytes = 3 * units * es  # v and a in, r out: the gate stream need never leave the chip
    gbs = alg_bytes * world * args.steps / (ms * 1e-3) / 1e9

    # each kernel alone, same rotation (the gate's output goes to the set's workspace)
    gviews = [s[2].view(tdt).view(gw.B, gw.L, gw.D) for s in sets]

    def gate_only(i):
        ssm.mhf_gate(sets[i % n_sets][1], tw, tb, gw.H, out=gviews[i % n_sets], stream=stream)

    def conv_only(i):
        ssm.causal_conv(sets[i % n_sets][0], gviews[i % n_sets], out=sets[i % n_sets][3], stream=stream)

    k_steps = max(10, min(args.steps, 500))
    for i in range(3):
        gate_only(i)
        conv_only(i)
    gate_us = timed(gate_only, k_steps) / k_steps * 1e3
    conv_us = timed(conv_only, k_steps) / k_steps * 1e3

    # end to end: pinned host v, a -> device, gated conv, r -> pinned host, every step
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    phv, pha = hv.pin_memory(), ha.pin_memory()
    phr = torch.empty_like(phv).pin_memory()
    dv_, da_, dws_, dr_ = sets[0]

    def e2e_step(_i):
        dv_.copy_(phv, non_blocking=True)
        da_.copy_(pha, non_blocking=True)
        ssm.mhf_gated_conv(dv_, da_, tw, tb, gw.H, out=dr_, workspace=dws_, stream=stream)
        phr.copy_(dr_, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    ems = timed(e2e_step, e2e_steps)
    e2e_gbs = alg_bytes * world * e2e_steps / (ems * 1e-3) / 1e9

    peak, peak_src = measured_peaks()
    C = gw.D // gw.H
    conv_bytes, gate_bytes = 3 * units * es, 2 * units * es + gw.D * C * gw.K * 4 + gw.D * 4
    gate_flops = 2 * units * C * gw.K * 3  # three fp16 products per term (hi*hi, hi*lo, lo*hi)
    kernel = "fftconv_fused_kernel" if gw.L <= 1024 else ("bigrow_group_kernel" if gw.L <= 4096 else "bigconv_kernel")
    dominant = (kernel, conv_bytes, conv_us) if conv_us >= gate_us else ("mhf_gate_kernel", gate_bytes, gate_us)
    traffic, _, _ = recorded_counters(gw.name, "mhf_gate_kernel")
    bf16_peak = None
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        bf16_peak = json.load(open(pp)).get("bf16_tflops")
    f16_peak = bf16_peak or 1590.0  # kind::f16 with fp16 operands runs at the bf16 rate
    line = {
        "metric": GATE_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": gw.name, "path": "gated", "B": gw.B, "L": gw.L, "D": gw.D, "heads": gw.H,
                   "taps": gw.K, "io_dtype": gw.dtype,
                   "l2": f"inputs larger than L2: {n_sets} rotating (v,a,g,r) sets of {set_bytes / 2 ** 20:.0f} MiB",
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "outputs_per_s": units * world * args.steps / (ms * 1e-3),
        "hbm_frac": gbs / world / peak,
        "roofline": {"bound": "hbm", "achieved": dominant[1] / (dominant[2] * 1e-6) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": dominant[1] / (dominant[2] * 1e-6) / 1e9 / peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "kernel": dominant[0],
                     "algorithmic_bytes_per_launch": dominant[1], "launch_us": dominant[2],
                     "traffic": None},
        "gate_kernel": {"kernel": "mhf_gate_kernel (tcgen05 kind::f16, 3 split products)", "launch_us": gate_us,
                        "hbm": {"achieved": gate_bytes / (gate_us * 1e-6) / 1e9, "peak": peak, "unit": "GB/s",
                                "frac": gate_bytes / (gate_us * 1e-6) / 1e9 / peak,
                                "algorithmic_bytes_per_launch": gate_bytes, "traffic": traffic},
                        "tensor": {"achieved": gate_flops / (gate_us * 1e-6) / 1e12, "peak": f16_peak,
                                   "unit": "TFLOP/s", "frac": gate_flops / (gate_us * 1e-6) / 1e12 / f16_peak,
                                   "flops_per_launch": gate_flops,
                                   "peak_source": "MEASURED_PEAKS.json bf16_tflops (fp16 runs at the bf16 rate)"}},
        "conv_kernel_us": conv_us,
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": 2 * units * es,
                "d2h_bytes_per_step": units * es, "steps": e2e_steps,
                "path": "pinned host v, a -> device; mhf_gated_conv; r -> pinned host"},
        "gpu_launches": args.steps * 2,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_ups, cores, desc, secs = gate_oracle_rate(gw, v if gw.dtype == "f32" else workloads.bf16_to_f32(v),
                                                      a if gw.dtype == "f32" else workloads.bf16_to_f32(a), w, bias,
                                                      budget_s=15.0)
        line["cpu_baseline"] = {"value": cpu_ups * 3 * es / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def run_gated_reference(args, rank, world):
    """The oracle (gate + direct sum) on the host cores, same metric."""
    if rank != 0:
        return
    gw = workloads.GATE_WORKLOADS[args.workload]
    v, a, w, bias = workloads.generate_gate(gw.B, gw.L, gw.D, gw.H, gw.K, "f32", gw.seed)
    per_step = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    import oracle
    import oracle.mhf_gate as mhf
    C = gw.D // gw.H
    sv, sa = np.ascontiguousarray(v[:1, :, :C]), np.ascontiguousarray(a[:1, :, :C])
    sw, sb = np.ascontiguousarray(w[:C]), np.ascontiguousarray(bias[:C])
    t0 = time.perf_counter()
    mhf.mhf_gated_conv(sv, sa, sw, sb, 1)
    reps = max(1, int(per_step / max(time.perf_counter() - t0, 1e-4)))
    for _ in range(args.warmup):
        mhf.mhf_gated_conv(sv, sa, sw, sb, 1)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(reps):
            mhf.mhf_gated_conv(sv, sa, sw, sb, 1)
    el = time.perf_counter() - t0
    es = 4 if gw.dtype == "f32" else 2
    units = gw.L * C * reps * args.steps
    gbs = units * 3 * es / el / 1e9
    sample = f"oracle (gate + direct sum) on head 0 of batch 0 of {gw.name}, {reps} passes per step"
    print(json.dumps({
        "impl": "reference", "metric": GATE_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": gw.name, "path": "gated", "B": gw.B, "L": gw.L, "D": gw.D, "heads": gw.H,
                   "taps": gw.K, "io_dtype": gw.dtype},
        "outputs_per_s": units / el,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_dwconv(args, rank, world, local):
    """The block's causal depthwise convolution: one step = one launch."""
    import torch
    import spectral_sequence_mixing_b200 as ssm

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    dw = workloads.DWCONV_WORKLOADS[args.workload]
    x, w, bias = workloads.generate_dwconv(dw.B, dw.L, dw.D, dw.K, dw.dtype, dw.seed + 1000 * rank)
    es = 4 if dw.dtype == "f32" else 2
    hx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if dw.dtype == "bf16" else torch.from_numpy(x)
    tw, tb = torch.from_numpy(w).to(dev), torch.from_numpy(bias).to(dev)
    units = dw.units
    set_bytes = 2 * units * es
    n_sets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    x0 = hx.to(dev)
    sets = [(x0 if i == 0 else x0.clone(), torch.empty_like(x0)) for i in range(n_sets)]
    stream = torch.cuda.current_stream(dev)

    def step(i):  # on the current stream (the capture stream inside a graph capture)
        sx, sy = sets[i % n_sets]
        ssm.causal_dwconv(sx, tw, tb, out=sy)

    def timed(fn, steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(steps):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), pg, dev)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    # A step (~8 us of device time) is shorter than a Python call through the
    # binding, so the steps are replayed from CUDA graphs: one graph of G
    # consecutive steps (whole rotations of the buffer sets) and one graph per
    # set for the remainder; every step is still one launch on its own buffers.
    G = n_sets * max(1, 64 // n_sets)
    big = torch.cuda.CUDAGraph()
    with torch.cuda.graph(big):
        for i in range(G):
            step(i)
    singles = []
    for k in range(n_sets):
        gk = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gk):
            step(k)
        singles.append(gk)
    torch.cuda.synchronize(dev)

    def run_steps(n):
        for _ in range(n // G):
            big.replay()
        for i in range(n % G):
            singles[i % n_sets].replay()

    run_steps(G)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    clocks = clk.report()
    ms_per_step = ms / args.steps
    alg_bytes = 2 * units * es + dw.D * (dw.K + 1) * 4
    gbs = alg_bytes * world * args.steps / (ms * 1e-3) / 1e9

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    phx = hx.pin_memory()
    phy = torch.empty_like(phx).pin_memory()
    dx_, dy_ = sets[0]

    def e2e_step(_i):
        dx_.copy_(phx, non_blocking=True)
        ssm.causal_dwconv(dx_, tw, tb, out=dy_)
        phy.copy_(dy_, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    ems = timed(e2e_step, e2e_steps)
    e2e_gbs = alg_bytes * world * e2e_steps / (ems * 1e-3) / 1e9
    peak, peak_src = measured_peaks()
    achieved = alg_bytes / (ms_per_step * 1e-3) / 1e9
    traffic, _, _ = recorded_counters(dw.name, "dwconv_vec_kernel")
    line = {
        "metric": DWCONV_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": dw.name, "path": "dwconv", "B": dw.B, "L": dw.L, "D": dw.D, "taps": dw.K,
                   "io_dtype": dw.dtype,
                   "l2": f"inputs larger than L2: {n_sets} rotating (x,y) sets of {set_bytes / 2 ** 20:.0f} MiB",
                   "launch": f"steps replayed from CUDA graphs ({G} steps per graph)",
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "outputs_per_s": units * world * args.steps / (ms * 1e-3),
        "hbm_frac": gbs / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "kernel": "dwconv_vec_kernel",
                     "algorithmic_bytes_per_launch": alg_bytes, "traffic": traffic},
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": units * es, "d2h_bytes_per_step": units * es,
                "steps": e2e_steps, "path": "pinned host x -> device; causal_dwconv; y -> pinned host"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        import oracle.mhf_dwconv as odw
        xf = workloads.bf16_to_f32(x) if dw.dtype == "bf16" else x
        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 15.0 and reps < 200:
            odw.causal_dwconv(xf, w, bias)
            reps += 1
        secs = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": units * reps * 2 * es / secs / 1e9, "unit": "GB/s",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"oracle (float64 numpy) on the whole {dw.name}, {reps} passes",
                                "seconds": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def run_dwconv_reference(args, rank, world):
    """The oracle (float64 numpy) on the host cores, same metric."""
    if rank != 0:
        return
    dw = workloads.DWCONV_WORKLOADS[args.workload]
    x, w, bias = workloads.generate_dwconv(dw.B, dw.L, dw.D, dw.K, "f32", dw.seed)
    import oracle
    import oracle.mhf_dwconv as odw
    for _ in range(args.warmup):
        odw.causal_dwconv(x, w, bias)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        odw.causal_dwconv(x, w, bias)
    el = time.perf_counter() - t0
    es = 4 if dw.dtype == "f32" else 2
    gbs = dw.units * args.steps * 2 * es / el / 1e9
    print(json.dumps({
        "impl": "reference", "metric": DWCONV_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": dw.name, "path": "dwconv", "B": dw.B, "L": dw.L, "D": dw.D, "taps": dw.K,
                   "io_dtype": dw.dtype},
        "outputs_per_s": dw.units * args.steps / el,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"oracle (float64 numpy) on the whole {dw.name} per step"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_probe(args, rank):
    """Time the rate probes of libccprobe.so (one warm-up launch, one timed
    launch each, CUDA events) with the SM clock sampled meanwhile, and report
    each as a rate per SM per clock and per second on the whole GPU."""
    import ctypes
    import torch
    if rank != 0:
        return
    from spectral_sequence_mixing_b200 import build as b
    b.build()
    lib = ctypes.CDLL(b.PROBE_LIB)
    lib.ccp_run.restype = ctypes.c_int
    lib.ccp_run.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double)]
    torch.cuda.init()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # (name, kind, blocks, threads, iters, unit)
    probes = [("ffma", 0, 2 * sms, 1024, 100000, "lane-op"), ("ffma2", 1, 2 * sms, 1024, 100000, "lane-op"),
              ("imad", 2, 2 * sms, 1024, 50000, "lane-op"), ("imad_hi", 3, 2 * sms, 1024, 50000, "lane-op"),
              ("smem_read", 4, 2 * sms, 1024, 10000, "byte"), ("dsmem_store_8cta", 5, (sms // 8) * 8, 512, 1000, "byte")]
    out = {}
    with ClockSampler(0) as clk:
        for name, kind, blocks, threads, iters, unit in probes:
            ms, units = ctypes.c_float(0), ctypes.c_double(0)
            st = lib.ccp_run(kind, blocks, threads, iters, ctypes.byref(ms), ctypes.byref(units))
            if st != 0:
                raise RuntimeError(f"probe {name}: CUDA error {st}")
            out[name] = {"ms": ms.value, "units": units.value, "unit": unit,
                         "sms_used": min(sms, blocks) if kind != 5 else blocks}
    clocks = clk.report()
    mhz = clocks["sm_mhz"] if clocks and clocks.get("sm_mhz") else 1965.0
    for name, r in out.items():
        per_s = r["units"] / (r["ms"] * 1e-3)
        r["per_s_gpu"] = per_s
        r["per_clk_per_sm"] = per_s / r["sms_used"] / (mhz * 1e6)
    print(json.dumps({"probe": out, "sm_count": sms, "clocks": clocks,
                      "note": "per_clk_per_sm at the median sampled SM clock"}), flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.probe:
        run_probe(args, rank)
        return
    if world != args.gpus and "RANK" in os.environ:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    gated = args.workload in workloads.GATE_WORKLOADS
    dwconv = args.workload in workloads.DWCONV_WORKLOADS
    if args.impl == "reference":
        (run_gated_reference if gated else run_dwconv_reference if dwconv else run_reference)(args, rank, world)
    elif gated:
        run_gated(args, rank, world, local)
    elif dwconv:
        run_dwconv(args, rank, world, local)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
