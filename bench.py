#!/usr/bin/env python
"""Benchmark of the block-scaled grouped GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bsg|reference] [--config I]
                    [--no-also] [--cpu-seconds S]

One step = one launch of the whole hot path (window scheduling, TMA loads, scale handling, tcgen05
MMAs, BF16 epilogue -- all inside one kernel) over one batch of synthetic input.  The headline
workload is the largest of the five, the NVFP4 grouped GEMM (G=8, M_g=8192, N=K=8192); `--config`
picks another.  The timed region is K back-to-back launches bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream, max over ranks.  Inputs are larger
than the 126 MB L2 for the headline workload (stated in the JSON `config`); smaller workloads flush
L2 between launches outside the per-launch events.

Rank 0 prints ONE JSON line (metric, value = whole-job TFLOPS, roofline of the kernel, the oracle's
CPU throughput on a bounded sample, the end-to-end number through host buffers, clocks sampled
during the timed region); on one GPU the line's `also` holds the same fields for each of the other
four workloads, and the activation quantisers' HBM throughput.  `--impl reference` times the fp64 CPU oracle on the same workload instead
(rank 0 only).  Under torchrun each rank runs its own copy of the workload on its own GPU (weak
scaling, no data-path collective: the op needs no exchange step).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "grouped block-scaled GEMM TFLOPS (FP8 & NVFP4) + % of B200 roofline"
# The headline workload: the largest of the five (NVFP4 grouped, G=8, M_g=8192, N=K=8192, 8.8 TFLOP);
# the metric names no single workload, so the largest one is the headline and the others are reported
# beside it with the same fields.
HEADLINE_CONFIG = 3
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal dense ratios to bf16 (2.25 PF): fp8 4.5 PF, fp4 9 PF
DTYPE_RATIO = {"fp8": 2.0, "nvfp4": 4.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["bsg", "reference"], default="bsg")
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG)
    ap.add_argument("--no-also", action="store_true", help="skip the other workloads' kernel numbers")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--sweep", action="store_true",
                    help="time every tactic on a set of shapes and compare with the chooser's pick")
    ap.add_argument("--moe-only", action="store_true",
                    help="time only the MoE expand permutation (three routing sizes)")
    ap.add_argument("--quant-only", action="store_true",
                    help="time only the activation quantisers (one JSON line each) -- for profiling")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- distributed helpers


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend, timeout_s=120):
    import datetime

    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ws, rank


def reduce_max(value, device=None):
    """Max of a float over ranks (the slowest rank sets the job time); identity when not distributed."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def job_value(per_rank_flops, max_seconds, world):
    """Whole-job throughput in TFLOPS: every rank processes its own (identical-size) batch."""
    return world * per_rank_flops / max_seconds / 1e12


# ----------------------------------------------------------------------------- peaks / clocks


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock, its maximum and the throttle reasons, sampled while the timed region runs.

    NVML (read-only queries) is polled every millisecond from a thread, so even a timed region of a
    few milliseconds gets samples; without NVML, nvidia-smi is polled every 100 ms."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.samples = []          # (sm_mhz, max_mhz, set of active reason names)
        self.source = None
        self.nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.masks = [(name, getattr(pynvml, attr, 0)) for name, attr in self.REASONS]
        except Exception:
            self.nvml = None

    def _poll_nvml(self):
        nv = self.nvml
        while not self.stop_flag.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
                self.samples.append((sm, self.max_mhz, {n for n, m in self.masks if m and bits & m}))
            except Exception:
                pass
            time.sleep(0.001)

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((sm, mx, {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}))

    def start(self):
        self.samples = []
        self.stop_flag.clear()
        if self.nvml is not None:
            self.source = "nvml, 1 ms"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.source = "nvidia-smi, 100 ms"
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.proc = None
        if self.thread:
            self.thread.join(timeout=2)
        if not self.samples:
            return None
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(x[0] for x in self.samples), "sm_max_mhz": self.samples[-1][1],
                "reasons": sorted(reasons), "samples": len(self.samples), "source": self.source}


def visible_gpu_index(local_rank):
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    if cvd:
        ids = [x.strip() for x in cvd.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ----------------------------------------------------------------------------- kernel source hash


# The device code each workload's counters depend on: its kernels' own headers, the shared PTX
# wrappers and scheduler, and the tactic chooser that picks among them.  A change anywhere else (host
# entry points, another kernel family, comments) leaves the recorded counters valid.
KERNEL_SOURCES = {
    "fp8": ["bsg_fp8.cuh", "bsg_fp8_swap.cuh", "bsg_sched.cuh", "bsg_ptx.cuh", "bsg_chooser.cpp"],
    "nvfp4": ["bsg_nvfp4.cuh", "bsg_sched.cuh", "bsg_ptx.cuh", "bsg_chooser.cpp"],
    "quant": ["bsg_quant.cuh"],
    "moe": ["bsg_moe.cuh"],
}


def kernel_family(workload_name):
    return workload_name.split("_", 1)[0]


def kernel_source_hash(family):
    """Hash of the code (comments and blank lines removed) of a kernel family's sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_grouped_gemm_indices_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[family]):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            code = [line.split("//", 1)[0].rstrip() for line in fh]
        h.update(f.encode())
        h.update("\n".join(line for line in code if line).encode())
    return h.hexdigest()[:16]


def recorded_profile(workload_name):
    """The committed ncu figures of one workload's kernel (profiles/traffic.json): DRAM bytes per
    launch and tensor-pipe activity, if taken on the current sources of that kernel; else {}."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload_name)
    if not e or e.get("source_hash") != kernel_source_hash(kernel_family(workload_name)):
        return {}
    return e


def recorded_traffic(workload_name):
    return recorded_profile(workload_name).get("bytes_per_launch")


# ----------------------------------------------------------------------------- our arm


class Runner:
    def __init__(self, w):
        import torch

        import nvfp4_grouped_gemm_indices_b200 as bsg
        self.bsg = bsg
        self.w = w
        dev = lambda x: None if x is None else torch.from_numpy(np.ascontiguousarray(x)).cuda()
        self.A, self.B, self.idx = dev(w.A), dev(w.B), dev(w.m_indices)
        if w.kind == "fp8":
            self.s1, self.s2, self.s3 = dev(w.a_scale), dev(w.b_scale), None
        else:
            self.s1, self.s2, self.s3 = dev(w.sfa), dev(w.sfb), dev(w.alpha)
        self.C = torch.zeros((w.M, w.N), dtype=torch.bfloat16, device="cuda")

    def tactic(self):
        """Name of the tactic the library's chooser picks for this workload."""
        w = self.w
        kind = 0 if w.kind == "fp8" else 1
        sms = torch_sm_count()
        return self.bsg.bsg_tactic_name(kind, self.bsg.bsg_choose_tactic(kind, w.M, w.N, w.K, w.G, sms))

    def launch(self, stream, A=None, B=None, s1=None, s2=None, s3=None, idx=None, C=None):
        w = self.w
        A = self.A if A is None else A
        B = self.B if B is None else B
        s1 = self.s1 if s1 is None else s1
        s2 = self.s2 if s2 is None else s2
        s3 = self.s3 if s3 is None else s3
        idx = self.idx if idx is None else idx
        C = self.C if C is None else C
        if w.kind == "fp8":
            self.bsg.bsg_fp8_grouped_gemm(A, B, s1, s2, idx, C, w.M, w.N, w.K, w.G, stream)
        else:
            self.bsg.bsg_nvfp4_gemm(A, B, s1, s2, s3, idx, C, w.M, w.N, w.K, w.G, stream)


def torch_sm_count():
    import torch
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def time_kernel(runner, steps, warmup, flush=None, sampler=None):
    """K back-to-back launches between synchronisations; returns (total seconds, mean per-launch
    seconds from per-launch event pairs on the launching stream, clocks sampled during the timed
    region or None)."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        runner.launch(stream.cuda_stream)
    torch.cuda.synchronize()
    runner.bsg.bsg_get_device_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    t0.record(stream)
    for i in range(steps):
        if flush is not None:
            flush()
        starts[i].record(stream)
        runner.launch(stream.cuda_stream)
        ends[i].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    barrier()
    runner.bsg.bsg_get_device_status()
    total = t0.elapsed_time(t1) / 1e3
    per = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / steps / 1e3
    return total, per, clocks


def time_e2e(runner, steps):
    """Host buffers in pinned memory: every step copies all operands host->device, runs the kernel
    through the C ABI and copies C back; timed with CUDA events on the stream."""
    import torch
    w = runner.w
    host = {}
    for name in ("A", "B", "s1", "s2", "s3", "idx"):
        t = getattr(runner, name)
        if t is not None:
            host[name] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            host[name].copy_(t.cpu())
    dev = {k: torch.empty_like(getattr(runner, k)) for k in host}
    Cdev = torch.empty_like(runner.C)
    Chost = torch.empty(runner.C.shape, dtype=runner.C.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = Chost.numel() * Chost.element_size()
    stream = torch.cuda.current_stream()

    def step():
        for k, t in host.items():
            dev[k].copy_(t, non_blocking=True)
        runner.launch(stream.cuda_stream, C=Cdev, **dev)
        Chost.copy_(Cdev, non_blocking=True)

    step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1) / 1e3 / steps, h2d, d2h


def make_flush():
    """L2 flush between timed launches: write a buffer of twice the L2 size, then read a second one
    of the same size, so the write's dirty lines are written back during the flush and not during the
    timed kernel (L2 starts cold and clean)."""
    import torch
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
    clean = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
    sink = torch.empty(1, dtype=torch.int64, device="cuda")

    def flush():
        buf.fill_(1)
        torch.sum(clean, dim=(0,), keepdim=True, out=sink)
    return flush


def roofline(w, per_launch_s, peaks, peak_src, sustained=False):
    bf16 = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    tensor_peak = bf16 * DTYPE_RATIO[w.kind]
    hbm = peaks["hbm_gbs"]
    flops = w.flops
    nbytes = w.algorithmic_bytes()
    t_tensor = flops / (tensor_peak * 1e12)
    t_hbm = nbytes / (hbm * 1e9)
    traffic = recorded_traffic(w.name)
    if t_hbm > t_tensor:
        ach = nbytes / per_launch_s / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": traffic, "algorithmic_bytes": nbytes,
                "peak_source": f"{peak_src} hbm_gbs (STREAM-style copy)"}
    ach = flops / per_launch_s / 1e12
    sustained_peak = peaks["bf16_tflops_sustained"] * DTYPE_RATIO[w.kind]
    return {"bound": "tensor", "achieved": round(ach, 1), "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
            "frac": round(ach / tensor_peak, 4), "frac_of_sustained_peak": round(ach / sustained_peak, 4),
            "traffic": traffic, "algorithmic_bytes": nbytes,
            "tensor_pipe_active_pct_ncu": recorded_profile(w.name).get("tensor_pipe_pct"),
            "peak_source": f"derived: {peak_src} bf16 {'sustained' if sustained else 'burst'} "
                           f"{peaks['bf16_tflops_sustained' if sustained else 'bf16_tflops']} TFLOP/s x "
                           f"{DTYPE_RATIO[w.kind]:g} ({w.kind} : bf16 nominal dense ratio); no {w.kind} "
                           f"peak is measured on this pool"}


def time_quantiser(kind, M, K, peaks, steps=50, warmup=5):
    """The step before the GEMM: BF16 activations [M, K], gathered through a random row permutation,
    quantised into the GEMM's A operand.  HBM-bound; returns the also-line dict."""
    import torch
    import nvfp4_grouped_gemm_indices_b200 as bsg
    g = torch.Generator(device="cuda").manual_seed(M + K)
    X = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    src = torch.randperm(M, device="cuda", generator=g).to(torch.int32)
    if kind == "fp8":
        A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        S = torch.empty((M, K // 128), dtype=torch.float32, device="cuda")
        launch = lambda st: bsg.bsg_quantize_fp8_rows(X, src, A, S, M, M, K, st)
        nbytes = 2 * M * K + M * K + 4 * M * (K // 128) + 4 * M
    else:
        gs = torch.tensor([float(X.float().abs().max()) / (448.0 * 6.0)], dtype=torch.float32, device="cuda")
        A = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        S = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
        launch = lambda st: bsg.bsg_quantize_nvfp4_rows(X, src, gs, A, S, M, M, K, st)
        nbytes = 2 * M * K + M * K // 2 + M * (K // 16) + 4 * M
    flush = make_flush() if 2 * M * K < 2 * L2_BYTES else None
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        launch(stream.cuda_stream)
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(steps):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        launch(stream.cuda_stream)
        b.record(stream)
        b.synchronize()
        tot += a.elapsed_time(b) / 1e3
    per = tot / steps
    ach = nbytes / per / 1e9
    return {"us_per_launch": round(per * 1e6, 2),
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach / peaks["hbm_gbs"], 4),
                         "traffic": recorded_traffic(f"quant_{kind}_rows_gather_m{M}_k{K}"),
                         "algorithmic_bytes": nbytes},
            "l2": "flushed" if flush else "inputs > L2"}


def time_moe_permute(T, top_k, G, peaks, steps=50, warmup=5):
    """The MoE expand permutation (one single-CTA launch up to 2^16 entries over at most 1024 experts,
    else three: per-tile counts, scan, stable scatter) on a Zipf-skewed routing of T tokens x top_k
    choices over G experts.  Integer work bound by the latency of its dependent steps; reported with
    the HBM bytes it must move, as GPU time per call (CUDA-graph replay of `steps` calls) and as the
    rate of calls issued one by one from Python."""
    import torch
    import nvfp4_grouped_gemm_indices_b200 as bsg
    g = torch.Generator(device="cuda").manual_seed(T * 131 + G)
    ranks = torch.arange(1, G + 1, dtype=torch.float64, device="cuda") ** -1.2
    ids = torch.multinomial((ranks / ranks.sum()).float(), T * top_k, replacement=True, generator=g)
    ids = ids.to(torch.int32).view(T, top_k)
    n = T * top_k
    need = bsg.bsg_moe_permute_workspace_size(T, top_k, G)
    ws = torch.empty(max(16, need), dtype=torch.uint8, device="cuda")
    outs = [torch.empty(n, dtype=torch.int32, device="cuda"), torch.empty(n, dtype=torch.int32, device="cuda"),
            torch.empty((T, top_k), dtype=torch.int32, device="cuda"),
            torch.empty(G + 1, dtype=torch.int32, device="cuda")]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        launch = lambda: bsg.bsg_moe_permute(ids, T, top_k, G, *outs, ws, ws.numel(), side.cuda_stream)
        for _ in range(warmup):
            launch()
        side.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(side)
        for _ in range(steps):
            launch()
        b.record(side)
        b.synchronize()
        per_host = a.elapsed_time(b) / 1e3 / steps
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for _ in range(steps):
                launch()
        graph.replay()
        side.synchronize()
        a.record(side)
        graph.replay()
        b.record(side)
        b.synchronize()
        per = a.elapsed_time(b) / 1e3 / steps
        del graph
    nbytes = 2 * 4 * n + 3 * 4 * n + 4 * (G + 1)      # ids read twice; src, m_indices, dst written
    return {"us_per_launch": round(per * 1e6, 2), "us_per_call_issued_from_python": round(per_host * 1e6, 2),
            "kernel_launches": 1 if need == 0 else 3,
            "hbm_bytes": nbytes, "achieved_gbs": round(nbytes / per / 1e9, 1),
            "note": "latency-bound integer work; GPU time per call from a CUDA graph of "
                    f"{steps} calls, inputs L2-resident"}


def cpu_baseline(w, seconds):
    """The oracle as it stands, on the host's cores, over a bounded sample of the workload's rows
    (all N columns each).  Returns (TFLOPS, cores, sample description)."""
    import oracle
    cores = oracle.max_threads()
    routed = np.nonzero((w.m_indices >= 0) & (w.m_indices < w.G))[0] if w.m_indices is not None \
        else np.arange(w.M)
    rng = np.random.default_rng(1234)
    # calibrate on one row per core
    probe = rng.choice(routed, size=min(cores, len(routed)), replace=False)
    t = time.perf_counter()
    run_oracle(w, probe)
    dt = time.perf_counter() - t
    per_row = dt / len(probe)
    n = int(max(len(probe), min(len(routed), seconds / max(per_row, 1e-9))))
    n = max(cores, (n // cores) * cores) if n >= cores else n
    rows = np.sort(rng.choice(routed, size=min(n, len(routed)), replace=False))
    t = time.perf_counter()
    run_oracle(w, rows)
    dt = time.perf_counter() - t
    flops = 2.0 * len(rows) * w.N * w.K
    return flops / dt / 1e12, cores, f"{len(rows)} random routed rows x all {w.N} columns ({dt:.1f} s)"


def run_oracle(w, rows, n_cols=None):
    import oracle
    if w.kind == "fp8":
        if n_cols is None:
            return oracle.fp8_grouped(w.A, w.B, w.a_scale, w.b_scale, w.m_indices, w.M, w.N, w.K, w.G, rows=rows)
        return oracle.fp8_grouped(w.A, w.B[:, :n_cols], w.a_scale, w.b_scale[:, :(n_cols + 127) // 128],
                                  w.m_indices, w.M, n_cols, w.K, w.G, rows=rows)
    if n_cols is None:
        return oracle.nvfp4(w.A, w.B, w.sfa, w.sfb, w.alpha, w.m_indices, w.M, w.N, w.K, w.G, rows=rows)
    return oracle.nvfp4(w.A, w.B[:, :n_cols], w.sfa, w.sfb[:, :n_cols], w.alpha, w.m_indices, w.M, n_cols, w.K,
                        w.G, rows=rows)


def needs_flush(w):
    """Inputs smaller than twice the L2 are flushed out of it between timed launches."""
    return (w.A.nbytes + w.B.nbytes) < 2 * L2_BYTES


def config_desc(w, cfg):
    """The workload, identically for both arms (sizes only; nothing that depends on the GPU)."""
    d = {"workload": w.name, "config_index": cfg, "kind": w.kind, "M": w.M, "N": w.N, "K": w.K, "G": w.G,
         "routed_rows": w.routed_rows, "active_experts": len(w.active_experts()),
         "input_bytes": int(w.A.nbytes + w.B.nbytes + (w.m_indices.nbytes if w.m_indices is not None else 0)),
         "parallelism": "replicas (one independent batch per GPU, no collective)"}
    d["l2"] = ("L2 flushed (2x126 MB written, then 2x126 MB read: cold and clean) between launches, outside the "
               "per-launch events" if needs_flush(w)
               else f"inputs {d['input_bytes'] / 1e6:.0f} MB > 126 MB L2, no flush")
    return d


def dtype_desc(w):
    return ("e4m3xe4m3->f32 (fp32 per-128 scales), bf16 out" if w.kind == "fp8"
            else "e2m1xe2m1 (ue4m3 per-16 scales)->f32, bf16 out")


def measure(w, cfg, steps, warmup, e2e_steps, cpu_seconds, peaks, peak_src, sampler, ws, rank):
    """Kernel time (device-resident inputs), end-to-end time through host buffers, and (rank 0 of a
    single-GPU run) the oracle's CPU throughput on a bounded sample, for one workload."""
    r = Runner(w)
    flush = make_flush() if needs_flush(w) else None
    total, per, clocks = time_kernel(r, steps, warmup, flush, sampler)
    if flush is not None:
        total = per * steps                 # the flushes between launches are not the kernel's time
    total = reduce_max(total, device="cuda")
    per = reduce_max(per, device="cuda")
    e2e_s, h2d, d2h = time_e2e(r, e2e_steps)
    e2e_s = reduce_max(e2e_s, device="cuda")
    out = {
        "value": round(job_value(w.flops, total / steps, ws), 2), "ms_per_step": round(total / steps * 1e3, 5),
        "us_per_launch": round(per * 1e6, 2), "tactic": r.tactic(), "config": config_desc(w, cfg),
        "roofline": roofline(w, per, peaks, peak_src), "clocks": clocks, "gpu_launches": steps,
        "e2e": {"value": round(job_value(w.flops, e2e_s, ws), 3), "unit": "TFLOPS", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "note": "all operands copied host->device from pinned memory and C copied back, every step"},
    }
    del r
    if ws == 1 and rank == 0:
        tf, cores, sample = cpu_baseline(w, cpu_seconds)
        out["cpu_baseline"] = {"value": tf, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample}
    return out


def run_bsg(args):
    import torch
    ws, rank, local = dist_env()
    if args.gpus != ws:
        if ws == 1 and args.gpus > 1:
            raise SystemExit("--gpus > 1 needs torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    init_dist("nccl")
    peaks, peak_src = load_peaks()

    sampler = ClockSampler(visible_gpu_index(local))
    from nvfp4_grouped_gemm_indices_b200 import workloads as W
    w = W.config(args.config)
    m = measure(w, args.config, args.steps, args.warmup, args.e2e_steps, args.cpu_seconds, peaks, peak_src,
                sampler, ws, rank)
    line = {
        "metric": METRIC, "value": m["value"], "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype_desc(w),
        "data": "synthetic (seeded; quantised N(0,1) activations, N(0,0.02) / N(0,1) weights)",
        "config": m["config"], "tactic": m["tactic"], "roofline": m["roofline"],
        "gpu_launches": m["gpu_launches"], "clocks": m["clocks"], "e2e": m["e2e"],
    }
    if "cpu_baseline" in m:
        line["cpu_baseline"] = m["cpu_baseline"]
    del w
    torch.cuda.empty_cache()
    if ws == 1 and rank == 0 and not args.no_also:
        also = {}
        for cfg in range(5):
            if cfg == args.config:
                continue
            wc = W.config(cfg)
            also[wc.name] = measure(wc, cfg, max(20, min(args.steps, 200)), max(3, args.warmup),
                                    min(args.e2e_steps, 10), max(4.0, args.cpu_seconds / 3), peaks, peak_src,
                                    sampler, ws, rank)
            del wc
            torch.cuda.empty_cache()
        also["quant_fp8_rows_gather_m8192_k7168"] = time_quantiser("fp8", 8192, 7168, peaks)
        also["quant_nvfp4_rows_gather_m65536_k8192"] = time_quantiser("nvfp4", 65536, 8192, peaks)
        also["moe_permute_t8192_k8_g64"] = time_moe_permute(8192, 8, 64, peaks)
        also["moe_permute_t64_k8_g64"] = time_moe_permute(64, 8, 64, peaks)
        also["moe_permute_t65536_k8_g256"] = time_moe_permute(65536, 8, 256, peaks)
        line["also"] = also
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from nvfp4_grouped_gemm_indices_b200 import workloads as W
    import oracle
    w = W.config(args.config)
    cores = oracle.max_threads()
    # per step: a bounded sample (rows x leading 128-column blocks) sized so that warmup + steps take
    # about 90 s of CPU time in total
    budget = 90.0 / max(1, args.steps + args.warmup)
    routed = np.nonzero((w.m_indices >= 0) & (w.m_indices < w.G))[0] if w.m_indices is not None \
        else np.arange(w.M)
    rng = np.random.default_rng(99)
    t = time.perf_counter()
    run_oracle(w, routed[:cores], n_cols=128)
    per_unit = (time.perf_counter() - t) / cores          # one row x 128 columns
    units = max(1, int(budget / max(per_unit, 1e-9)))
    rows_per_step = max(1, min(cores, units))
    cols = int(min(w.N, max(128, 128 * (units // rows_per_step)))) // 128 * 128
    for _ in range(args.warmup):
        run_oracle(w, rng.choice(routed, rows_per_step, replace=False), n_cols=cols)
    t = time.perf_counter()
    for _ in range(args.steps):
        run_oracle(w, rng.choice(routed, rows_per_step, replace=False), n_cols=cols)
    dt = (time.perf_counter() - t) / args.steps
    flops = 2.0 * rows_per_step * cols * w.K
    value = flops / dt / 1e12
    sample = f"per step {rows_per_step} random routed rows x the first {cols} columns of {w.name}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (decoded operands; " + dtype_desc(w) + " inputs)",
        "data": "synthetic (seeded; quantised N(0,1) activations, N(0,0.02) / N(0,1) weights)",
        "config": config_desc(w, args.config),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_quant_only(args):
    import torch
    torch.cuda.set_device(0)
    peaks, _ = load_peaks()
    for kind, M, K in (("fp8", 8192, 7168), ("nvfp4", 65536, 8192)):
        d = time_quantiser(kind, M, K, peaks, steps=max(1, args.steps), warmup=max(1, args.warmup))
        print(json.dumps({"kernel": f"quant_{kind}_rows_gather_m{M}_k{K}", **d}), flush=True)


def run_moe_only(args):
    import torch
    torch.cuda.set_device(0)
    peaks, _ = load_peaks()
    for T, top_k, G in ((8192, 8, 64), (64, 8, 64), (65536, 8, 256)):
        d = time_moe_permute(T, top_k, G, peaks, steps=max(1, args.steps), warmup=max(1, args.warmup))
        print(json.dumps({"kernel": f"moe_permute_t{T}_k{top_k}_g{G}", **d}), flush=True)


def sweep_shapes():
    """The five workloads plus shapes that move the pick: few rows over many experts, a dense tail,
    skewed and balanced routings."""
    from nvfp4_grouped_gemm_indices_b200 import workloads as W
    rng = np.random.default_rng(7)
    out = [W.config(i) for i in range(5)]
    for (M, N, K, G) in [(2048, 4096, 7168, 8), (4096, 2048, 4096, 16), (1024, 7168, 2048, 32), (16384, 4096, 4096, 4)]:
        idx = W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G))
        out.append(W.make_fp8(M, N, K, G, idx, seed=M + N, name=f"fp8_sweep_g{G}_m{M}_n{N}_k{K}"))
    # the FP8 page's two benchmark shapes (small launches)
    for (M, N, K, G) in [(65, 128, 128, 2), (777, 256, 512, 8)]:
        counts = [M // G + (1 if i < M % G else 0) for i in range(G)]
        out.append(W.make_fp8(M, N, K, G, W.counts_to_indices(counts), seed=M, name=f"fp8_page_g{G}_m{M}_n{N}_k{K}"))
    # few rows per expert (decode): where the operand-swapped tiles take over from the row tiles
    idx = W.routing_zipf(96, 32, rng)
    out.append(W.make_fp8(96, 2048, 4096, 32, idx, seed=96, name="fp8_sweep_zipf_g32_m96_n2048_k4096"))
    for (M, N, K, G) in [(256, 4096, 2048, 16), (512, 4096, 4096, 8), (1024, 4096, 4096, 8)]:
        idx = W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G))
        out.append(W.make_fp8(M, N, K, G, idx, seed=M + N + G, name=f"fp8_sweep_g{G}_m{M}_n{N}_k{K}"))
    for (M, N, K, G) in [(1024, 8192, 4096, 1), (8192, 4096, 4096, 8), (512, 16384, 8192, 4)]:
        idx = W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G))
        out.append(W.make_nvfp4(M, N, K, G, idx, seed=M + N, name=f"nvfp4_sweep_g{G}_m{M}_n{N}_k{K}"))
    return out


def run_sweep(args):
    """Every tactic on every sweep shape: prints one JSON line per shape with the time of each tactic,
    the chooser's pick and its regret (time of the pick / best time)."""
    import torch
    import nvfp4_grouped_gemm_indices_b200 as bsg
    torch.cuda.set_device(0)
    sms = torch_sm_count()
    regrets = []
    for w in sweep_shapes():
        kind = 0 if w.kind == "fp8" else 1
        r = Runner(w)
        flush = make_flush() if (w.A.nbytes + w.B.nbytes) < 2 * L2_BYTES else None
        times = {}
        for t in range(bsg.bsg_num_tactics(kind)):
            bsg.bsg_set_tactic(kind, t)
            _, per, _ = time_kernel(r, max(10, min(args.steps, 100)), 3, flush)
            times[bsg.bsg_tactic_name(kind, t)] = per
        bsg.bsg_set_tactic(kind, -1)
        pick = bsg.bsg_tactic_name(kind, bsg.bsg_choose_tactic(kind, w.M, w.N, w.K, w.G, sms))
        best = min(times, key=times.get)
        regret = times[pick] / times[best]
        regrets.append(regret)
        print(json.dumps({"shape": w.name, "us": {k: round(v * 1e6, 2) for k, v in times.items()},
                          "chooser": pick, "best": best, "regret": round(regret, 4)}), flush=True)
        del r
        torch.cuda.empty_cache()
    print(json.dumps({"shapes": len(regrets), "picks_best": sum(1 for x in regrets if x == 1.0),
                      "geomean_regret": round(float(np.exp(np.mean(np.log(regrets)))), 4),
                      "max_regret": round(max(regrets), 4)}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.sweep:
        run_sweep(args)
        return
    if args.quant_only:
        run_quant_only(args)
        return
    if args.moe_only:
        run_moe_only(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_bsg(args)
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
