#!/usr/bin/env python
"""Benchmark of the block-scaled int8 projection on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0).  A *step* is one pass of the projection path
over one batch of synthetic input with the requantised weight resident (the
weight requantisation runs once, before timing, as the launcher page's
``ensure_int8_weight`` does):

* ``decode`` (M=1, N=K=4096, the default): one launch of the decode kernel
  (activation requantisation fused, CUDA cores); metric HBM GB/s over the
  algorithmic bytes N*K + N*K/8 + 2*M*K + 2*M*N.
* ``ffn_up`` / ``ffn_down`` / ``square_ragged``: requant_a + tcgen05 GEMM;
  metric TOPS = 2*M*N*K / step time (requantisation included).

Decode: the K timed steps are one CUDA-graph replay, each step on a different
copy of the requantised weight (copies cover >= 3x L2), timed with CUDA events
around the replay.  Prefill: L2 is flushed (a 256 MiB device write) before
every timed step, outside the per-step CUDA events.  ``ms_per_step`` is the
mean step time.
``e2e`` repeats the step through the public API with the activations moved
in from pinned host memory and the output moved back inside the events: for
decode through ``bsr_decode_host`` (copy kernels chained with the decode
kernel), for prefill through ``bsr_proj_host`` (row chunks whose copies in
and out overlap the neighbouring chunks' requantisation and GEMM).
Under torchrun every rank runs the same workload on its own GPU (independent
replicas: the path has no exchange step), timings are max-reduced over ranks.
``--impl reference`` times the CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
INT8_NOMINAL_TOPS = 4500.0  # B200 dense int8 tensor figure (datasheet), for context beside the measured peak
FP4_PER_BF16 = 4.0  # nominal dense FP4 / bf16 tensor ratio on B200 (9 / 2.25 PFLOP/s)
ORACLE_MAX_WORKERS = 16  # host processes of the all-cores oracle baseline
# The exact per-block rescale costs 2 FP32 FMAs per output element and 32-wide
# K block (= 64 int8 ops); the FP32 pipe retires 128 FMAs per clock per SM.
OPS_PER_SM_CLOCK_FMA_BOUND = 64 * 128 / 2


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="decode", choices=["decode", "ffn_up", "ffn_down", "square_ragged"])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-extra", action="store_true", help="skip the secondary prefill measurements")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle baseline sample")
    p.add_argument("--no-cpu", action="store_true", help="skip the oracle baseline (profiling runs)")
    p.add_argument("--only", default=None,
                   choices=["decode", "proj", "gemm", "requant_a", "requant_w", "requant_silu_a", "w4a16", "w4a4_decode"],
                   help="time one operation of the path alone on the workload (for profiling) and print its line")
    return p.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; timing max-reduced over ranks)
# ---------------------------------------------------------------------------


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def dist_init(backend: str):
    rank, world, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def dist_max(values, device="cpu"):
    """Element-wise max over ranks of a list of floats (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def dist_sum(values, device="cpu"):
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.cpu().tolist()


def dist_finish():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# peaks, clocks, roofline
# ---------------------------------------------------------------------------


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = [
        ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
        ("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
        ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
        ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
        ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
        ("applications_clocks_setting", "nvmlClocksEventReasonApplicationsClocksSetting"),
    ]

    def __init__(self, pci_bus_id: str | None, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(pci_bus_id) if pci_bus_id else pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks stay unknown
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            self._sample_once()
            time.sleep(self.period)

    def _sample_once(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, const in self.REASONS:
                if r & getattr(self.nv, const, 0):
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.nv is not None:
            self._sample_once()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        if self.nv is not None:
            self._sample_once()

    def summary(self):
        return {
            "sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
            "sm_max_mhz": float(self.max_mhz) if self.max_mhz else None,
            "reasons": sorted(self.reasons),
            "samples": len(self.samples),
        }


def measure_int8_peak(device, n=8192, reps=10):
    """Dense int8 tensor throughput of this GPU in TOPS: torch._int_mm (cuBLAS
    int8 GEMM, int32 out) of n x n x n, best of `reps` launches timed with
    CUDA events on the current stream."""
    import torch

    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device).t()  # column-major operand
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / (best / 1e3) / 1e12


def host_cpu():
    """CPU model and logical core count of the host running the oracle."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return {"model": model, "nproc": usable}


def roofline(bound, achieved, peak, unit, traffic):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": (achieved / peak) if peak else None, "traffic": traffic}


# translation unit of each measured kernel; with the csrc headers it includes
# and the C-ABI layer that picks its launch parameters, these are the sources
# its DRAM traffic depends on
KERNEL_UNITS = {"decode_kernel": "decode.cu", "gemm_kernel": "gemm_tc.cu", "requant_a_kernel": "requant.cu",
                "requant_w_kernel": "requant.cu", "requant_silu_a_kernel": "silu.cu",
                "nvfp4_gemv_kernel": ("nvfp4_gemv.cu", "w4a4.cu")}
LAUNCH_LAYER = "api.cu"


def _csrc_dir():
    return os.path.join(ROOT, "block_scaled_precision_requant_b200", "csrc")


def kernel_sources(kernel: str):
    """Sorted csrc file names that the kernel's code and launch depend on:
    its translation unit, the launch layer, and every csrc header they
    include, transitively."""
    csrc = _csrc_dir()
    unit = KERNEL_UNITS[kernel]
    todo = [*(unit if isinstance(unit, tuple) else (unit,)), LAUNCH_LAYER]
    seen = set()
    while todo:
        name = todo.pop()
        if name in seen or not os.path.exists(os.path.join(csrc, name)):
            continue
        seen.add(name)
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            todo += re.findall(r'^\s*#\s*include\s+"([^"]+)"', f.read(), flags=re.M)
    return sorted(seen)


def kernel_source_hash(kernel: str):
    """Hash of the kernel's sources (kernel_sources) with comments and
    whitespace removed: stored ncu traffic counts are valid only for this
    code.  Files the kernel does not depend on do not enter it."""
    h = hashlib.sha256()
    csrc = _csrc_dir()
    for name in kernel_sources(kernel):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # block comments
        text = re.sub(r"//[^\n]*", " ", text)  # line comments (no source string holds //)
        text = " ".join(text.split())
        h.update(name.encode())
        h.update(text.encode())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from profiles/dram_traffic.txt (lines:
    ``<kernel> <workload> <source-hash> <bytes>``), or None when absent or
    taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    src = kernel_source_hash(kernel) if kernel in KERNEL_UNITS else None
    for line in lines:
        parts = line.split()
        if len(parts) == 4 and parts[0] == kernel and parts[1] == workload and parts[2] == src:
            return float(parts[3])
    return None


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


def workload_desc(wl, world=1):
    """The `config` object of the bench line: the same for both arms."""
    m, n, k = wl.shape
    l2 = ("rotating copies of the requantised weight covering >= 3x L2 across the K steps of one CUDA-graph replay"
          if m <= 16 else "flushed before every timed step (256 MiB device write, outside the step events)")
    return {"workload": f"{wl.name}: M={m} N={n} K={k} (NVFP4 weight, BF16 activations '{wl.act}')",
            "m": m, "n": n, "k": k, "seed": wl.seed, "l2": l2,
            "parallelism": f"replicas x{world} (no exchange step)"}


def input_hashes(d):
    """SHA-256 of every input buffer of a generated workload (the NVFP4
    weight's nibbles and E4M3 bytes, its F32 scale2, the BF16 activations)."""
    from block_scaled_precision_requant_b200 import synth

    return {"w_packed": synth.sha256(d["w_packed"]), "w_e4m3": synth.sha256(d["w_e4m3"]),
            "scale2": synth.sha256(np.asarray(d["scale2"], dtype=np.float32)), "a_bf16": synth.sha256(d["a_bits"])}


def decode_bytes(m, n, k):
    """Algorithmic HBM bytes of one decode step: int8 weight, its F32 scales
    (4 B per 32), BF16 activations in, BF16 outputs out."""
    return n * k + n * (k // 32) * 4 + 2 * m * k + 2 * m * n


def prefill_ops(m, n, k):
    return 2 * m * n * k


def fma_bound_tops(num_sms, sm_mhz):
    """int8 ops/s of the GEMM when the FP32 pipe does nothing but the exact
    rescale (2 FMAs per element and 32-block), in TOPS."""
    return OPS_PER_SM_CLOCK_FMA_BOUND * num_sms * sm_mhz * 1e6 / 1e12


class Gpu:
    """Device state of one workload: requantised weight resident in HBM."""

    def __init__(self, name, device):
        import torch

        from block_scaled_precision_requant_b200 import synth

        import block_scaled_precision_requant_b200 as bsr

        self.torch, self.bsr = torch, bsr
        self.wl = synth.WORKLOADS[name]
        d = synth.make_workload(name)
        self.host = d
        m, n, k = self.wl.shape
        self.dev = device
        self.num_sms = torch.cuda.get_device_properties(device).multi_processor_count
        wp = torch.from_numpy(d["w_packed"]).to(device)
        we = torch.from_numpy(d["w_e4m3"]).to(device)
        self.w_i8, self.w_s = bsr.requant_w(wp, we, float(d["scale2"]))
        self.wp, self.we = wp, we
        self.a = torch.from_numpy(d["a_bits"].view(np.int16)).view(torch.bfloat16).to(device)
        self.out = torch.empty((m, n), dtype=torch.bfloat16, device=device)
        need = bsr.proj_scratch_bytes(m, k)
        self.scratch = torch.empty((max(need, 1),), dtype=torch.uint8, device=device)
        if m > bsr.DECODE_MAX_M:
            self.a_i8, self.a_st = bsr.requant_a(self.a)
        self.flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=device)
        self.a_host = torch.from_numpy(d["a_bits"].view(np.int16)).view(torch.bfloat16).pin_memory()
        self.out_host = torch.empty((m, n), dtype=torch.bfloat16).pin_memory()
        torch.cuda.synchronize()

    def step(self):
        self.bsr.proj(self.a, self.w_i8, self.w_s, self.out, self.scratch if self.scratch.numel() > 1 else None)

    def step_e2e(self):
        m = self.wl.shape[0]
        if m <= self.bsr.DECODE_MAX_M:
            self.bsr.decode_host(self.a_host, self.w_i8, self.w_s, self.out_host, self.a, self.out)
            return
        # 512-row chunks: the best of 256 / 512 / 1024 / 2048 / the default on
        # the three prefill shapes together
        self.bsr.proj_host(self.a_host, self.w_i8, self.w_s, self.out_host, self.a, self.out, self.scratch, 512)

    def launches_per_step(self):
        m, _, k = self.wl.shape
        return 1 if (m <= self.bsr.DECODE_MAX_M or k % 128) else 2

    def timed_graph_rotating(self, steps, warmup):
        """Device time of `steps` back-to-back steps captured in one CUDA graph,
        each step on a different copy of the requantised weight (copies cover
        at least 3x L2, so no step finds its weight in L2); returns per-step
        times (ms) as `steps` equal shares of the replay."""
        torch = self.torch
        l2 = torch.cuda.get_device_properties(self.dev).L2_cache_size
        wbytes = self.w_i8.numel() + 4 * self.w_s.numel()
        copies = max(2, -(-3 * l2 // wbytes))
        ws = [(self.w_i8.clone(), self.w_s.clone()) for _ in range(copies)]
        bsr = self.bsr
        # the weight copies are written before the capture and never inside
        # it, so every step may start its weight stream before the previous
        # step ends (the static-weight decode option)
        for i in range(max(warmup, 1)):  # eager warm-up also fills the launch caches
            w, s = ws[i % copies]
            bsr.decode(self.a, w, s, self.out, static_weight=True)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                w, s = ws[i % copies]
                bsr.decode(self.a, w, s, self.out, static_weight=True)
        g.replay()  # warm replay
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        total = e0.elapsed_time(e1)
        self.rotating_copies = copies
        del g, ws
        return [total / steps] * steps

    def timed_e2e_graph(self, steps, warmup):
        """End to end through the public API as a decode loop runs it: every
        step reads its activations from pinned host memory, runs the decode
        kernel and writes the result back to pinned host memory
        (``bsr_decode_host``: copy kernels chained with the decode kernel);
        the K steps are captured in one CUDA graph (so the host's Python
        overhead is not what is measured) over rotating weight copies
        (>= 3x L2)."""
        torch, bsr = self.torch, self.bsr
        l2 = torch.cuda.get_device_properties(self.dev).L2_cache_size
        wbytes = self.w_i8.numel() + 4 * self.w_s.numel()
        copies = max(2, -(-3 * l2 // wbytes))
        ws = [(self.w_i8.clone(), self.w_s.clone()) for _ in range(copies)]

        def one(i):
            w, s = ws[i % copies]
            bsr.decode_host(self.a_host, w, s, self.out_host, self.a, self.out, static_weight=True)

        for i in range(max(warmup, 1)):
            one(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                one(i)
        g.replay()
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        total = e0.elapsed_time(e1)
        del g, ws
        return [total / steps] * steps

    def timed(self, fn, steps, warmup, events_inside=None):
        """Per-step CUDA-event times (ms) of fn, L2 flushed before each step.
        events_inside(i) may return (start, end) events of the dominant kernel."""
        torch = self.torch
        for _ in range(warmup):
            self.flush.zero_()
            fn()
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            self.flush.zero_()
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        dist_barrier()
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in ev]

    def timed_gemm_only(self, steps, warmup):
        """Events around the tensor-core GEMM alone (its own launch, same stream)."""
        bsr = self.bsr
        fn = lambda: bsr.gemm(self.a_i8, self.a_st, self.w_i8, self.w_s, self.out)
        return self.timed(fn, steps, warmup)

    def timed_requant_a_only(self, steps, warmup):
        bsr = self.bsr
        fn = lambda: bsr.requant_a(self.a, self.a_i8, self.a_st)
        return self.timed(fn, steps, warmup)

    def timed_requant_w_only(self, steps, warmup):
        bsr = self.bsr
        fn = lambda: bsr.requant_w(self.wp, self.we, float(self.host["scale2"]), self.w_i8, self.w_s)
        return self.timed(fn, steps, warmup)

    def check_status(self):
        st = self.bsr.device_status()
        if st != 0:
            raise RuntimeError(f"device status word {st}: a pipeline wait timed out")


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------


_POOL_W = None


def _pool_init(w_i8, w_s):
    """Worker start-up of the all-cores oracle: keep the requantised weight."""
    global _POOL_W
    _POOL_W = (w_i8, w_s)


def _pool_rows(a_rows):
    """One oracle projection of the given activation rows (in a worker)."""
    import oracle

    oracle.proj_rows(a_rows, *_POOL_W)
    return len(a_rows)


class OracleRunner:
    """Times the CPU oracle on a bounded sample of a workload.  The weight
    requantisation runs once, outside the timing (as on the GPU)."""

    def __init__(self, name):
        import oracle
        from block_scaled_precision_requant_b200 import synth

        self.oracle = oracle
        self.wl = synth.WORKLOADS[name]
        d = synth.make_workload(name)
        m, n, k = self.wl.shape
        self.w_i8, self.w_s = oracle.requant_w(d["w_packed"], d["w_e4m3"], d["scale2"], k)
        self.a = d["a_bits"]
        self.rows = synth.sample_rows(m, min(m, 64), self.wl.seed)
        self.hashes = input_hashes(d)

    def sample_step(self, nrows):
        """Oracle projection of `nrows` sampled rows; returns seconds."""
        t0 = time.perf_counter()
        self.oracle.proj_rows(self.a[self.rows[:nrows]], self.w_i8, self.w_s)
        return time.perf_counter() - t0

    def per_row_seconds(self, budget_s):
        """Mean oracle seconds per activation row on one core, over a sample
        bounded by budget_s."""
        done, spent = 0, 0.0
        while spent < budget_s and done < 1000:
            spent += self.sample_step(1)
            done += 1
        return spent / done, done

    def per_row_seconds_all_cores(self, single_row_s, budget_s):
        """Wall seconds per activation row with the sampled rows spread over
        host worker processes (spawned, one per core up to
        ORACLE_MAX_WORKERS): the oracle unchanged, run side by side.
        Returns (seconds per row, rows, workers)."""
        import multiprocessing

        workers = max(1, min(host_cpu()["nproc"], ORACLE_MAX_WORKERS))
        per_worker = max(1, int(budget_s / max(single_row_s, 1e-6)))
        nrows = workers * per_worker
        tasks = [self.a[self.rows[i % len(self.rows)]][None] for i in range(nrows)]
        ctx = multiprocessing.get_context("spawn")
        with ctx.Pool(workers, initializer=_pool_init, initargs=(self.w_i8, self.w_s)) as pool:
            pool.map(_pool_rows, tasks[:workers], chunksize=1)  # warm-up: every worker once
            t0 = time.perf_counter()
            pool.map(_pool_rows, tasks, chunksize=per_worker)
            wall = time.perf_counter() - t0
        return wall / nrows, nrows, workers


def units_per_step(wl):
    m, n, k = wl.shape
    if m <= 16:
        return decode_bytes(m, n, k) / 1e9, "GB/s", "int8 block-scaled proj HBM GB/s (M=1 decode, incl. requant)"
    return prefill_ops(m, n, k) / 1e12, "TOPS", "int8 block-scaled proj TOPS (prefill, incl. requant)"


def cpu_baseline(name, budget_s, all_cores=True):
    """The oracle as it stands on the host: one core, and the same rows
    spread over worker processes on all cores (up to ORACLE_MAX_WORKERS).
    Step time = time per activation row x M (extrapolated when M > 1)."""
    r = OracleRunner(name)
    per_row, rows = r.per_row_seconds(budget_s)
    units, unit, _ = units_per_step(r.wl)
    m = r.wl.m
    ext = " (extrapolated)" if m > 1 else ""
    host = host_cpu()
    res = {"value": units / (per_row * m), "unit": unit, "cores": 1, "kind": "oracle",
           "sample": (f"{rows} oracle projection(s) of one sampled activation row each against the full requantised "
                      f"weight on one core; step time = per-row time x M={m}{ext}"),
           "ms_per_step": per_row * m * 1e3, "cpu_model": host["model"], "nproc": host["nproc"]}
    if all_cores:
        per_row_p, prow, workers = r.per_row_seconds_all_cores(per_row, budget_s / 2)
        res["all_cores"] = {"value": units / (per_row_p * m), "unit": unit, "cores": workers,
                            "ms_per_step": per_row_p * m * 1e3,
                            "sample": (f"{prow} sampled rows over {workers} spawned worker processes (wall time); "
                                       f"step time = wall time per row x M={m}{ext}")}
    return res


def reference_main(args):
    """The reference arm: the CPU oracle as it stands, on the host cores, on
    the GPU arm's workload, metric and unit.  Each step projects one sampled
    activation row per worker process (spawned, one per core up to
    ORACLE_MAX_WORKERS) against the full requantised weight; step time = wall
    time per row x M."""
    import multiprocessing

    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from block_scaled_precision_requant_b200 import synth

    wl = synth.WORKLOADS[args.workload]
    r = OracleRunner(args.workload)
    units, unit, metric = units_per_step(wl)
    host = host_cpu()
    workers = max(1, min(host["nproc"], ORACLE_MAX_WORKERS))
    rows = [r.a[r.rows[i % len(r.rows)]][None] for i in range(workers)]
    ctx = multiprocessing.get_context("spawn")
    with ctx.Pool(workers, initializer=_pool_init, initargs=(r.w_i8, r.w_s)) as pool:
        for _ in range(args.warmup):
            pool.map(_pool_rows, rows, chunksize=1)
        t = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            pool.map(_pool_rows, rows, chunksize=1)
            t.append((time.perf_counter() - t0) / workers)
    step_s = float(np.mean(t)) * wl.m
    value = units / step_s
    sample = (f"each step: {workers} sampled activation rows, one per worker process, against the full requantised "
              f"weight; step time = wall time per row x M={wl.m}" + (" (extrapolated)" if wl.m > 1 else ""))
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded generator; no dataset or trained weights)",
            "impl": "reference",
            "config": {**workload_desc(wl, args.gpus), "inputs_sha256": r.hashes},
            "cpu_baseline": {"value": value, "unit": unit, "cores": workers, "kind": "oracle", "sample": sample,
                             "cpu_model": host["model"], "nproc": host["nproc"]},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------


def mean_ms(times):
    return float(np.mean(times))


def prefill_extra(name, device, steps, warmup, peaks, int8_peak, pci, cpu=True, cpu_budget=6.0):
    """Full measurement record of one prefill workload (rank-local): the step
    (requant_a + GEMM), the GEMM alone with its roofline, the two
    requantisations, clocks sampled during the GEMM timing, the end-to-end
    step through the public API, and the oracle baseline."""
    g = Gpu(name, device)
    m, n, k = g.wl.shape
    ops = prefill_ops(m, n, k)
    t_step = mean_ms(g.timed(g.step, steps, warmup))
    with ClockSampler(pci) as clk:
        t_gemm = mean_ms(g.timed_gemm_only(steps, warmup))
    t_ra = mean_ms(g.timed_requant_a_only(steps, warmup))
    t_rw = mean_ms(g.timed_requant_w_only(steps, warmup))
    t_e2e = mean_ms(g.timed(g.step_e2e, max(3, steps // 2), 1))
    g.check_status()
    clocks = clk.summary()
    mhz = clocks["sm_mhz"] or peaks["sm_max_mhz"]
    fma_peak = fma_bound_tops(g.num_sms, mhz)
    achieved = ops / t_gemm / 1e9
    rl = roofline("alu", achieved, fma_peak, "TOPS", stored_traffic("gemm_kernel", name))
    rl.update({
        "kernel": "gemm_kernel", "tile_m": g.bsr.gemm_block_m(m, n),
        "peak_source": (f"2 FP32 FMAs per element and 32-block at 128 FMA/clk/SM x {g.num_sms} SMs x {mhz:g} MHz "
                        f"(median SM clock sampled during the GEMM timing)"),
        "tensor_peak": int8_peak, "tensor_frac": achieved / int8_peak,
        "tensor_peak_source": "torch._int_mm int8 8192^3, best of 10, measured in this run",
        "tensor_peak_nominal": INT8_NOMINAL_TOPS, "tensor_frac_nominal": achieved / INT8_NOMINAL_TOPS,
    })
    ra_gbs = m * k * 3.125 / t_ra / 1e6
    rw_gbs = n * k * 1.6875 / t_rw / 1e6
    res = {
        "shape": [m, n, k],
        "tops_incl_requant": ops / t_step / 1e9,
        "ms_step": t_step,
        "roofline": rl,
        "requant_a": {"gbs": ra_gbs, "frac_of_hbm": ra_gbs / peaks["hbm_gbs"], "ms": t_ra,
                      "bytes": m * k * 3.125, "traffic": stored_traffic("requant_a_kernel", name)},
        "requant_w": {"gbs": rw_gbs, "frac_of_hbm": rw_gbs / peaks["hbm_gbs"], "ms": t_rw,
                      "bytes": n * k * 1.6875, "traffic": stored_traffic("requant_w_kernel", name)},
        "clocks": clocks,
        "e2e": {"value": ops / t_e2e / 1e9, "unit": "TOPS", "h2d_bytes_per_step": 2 * m * k,
                "d2h_bytes_per_step": 2 * m * n, "ms_per_step": t_e2e,
                "how": "eager calls per step through bsr_proj_host (pinned host activations in and output out in "
                       "row chunks, the copies overlapped with the neighbouring chunks' requant_a + GEMM)"},
    }
    if g.wl.act == "silu_mul":
        res["silu"] = silu_extra(g, steps, warmup, cpu)
    del g
    import torch

    torch.cuda.empty_cache()
    if cpu:
        res["cpu_baseline"] = cpu_baseline(name, cpu_budget)
    return res


def w4a4_gemm_extra(device, steps, warmup, peaks):
    """The W4A4 projection on the tensor cores (block-scaled FP4 MMA) on the
    2048 x 14336 x 4096 shape with the FFN-up inputs: the composite entry
    (row quantiser, scale relayout, GEMM) and the GEMM alone, against the FP4
    tensor figure (measured bf16 peak x the nominal FP4/bf16 ratio)."""
    import torch

    import block_scaled_precision_requant_b200 as bsr
    from block_scaled_precision_requant_b200 import synth

    d = synth.make_workload("ffn_up")
    m, n, k = d["workload"].shape
    wp = torch.from_numpy(d["w_packed"]).to(device)
    w_sf = bsr.sf_blocked(torch.from_numpy(d["w_e4m3"]).to(device))
    a = torch.from_numpy(d["a_bits"].view(np.int16)).view(torch.bfloat16).to(device)
    s2 = float(d["scale2"])
    out = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    scratch = torch.empty((bsr.w4a4_proj_scratch_bytes(m, k),), dtype=torch.uint8, device=device)
    ap, ae, as2 = bsr.quant_nvfp4_rows(a)
    a_sf = bsr.sf_blocked(ae)
    status = torch.zeros((1,), dtype=torch.int32, device=device)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=device)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.mean(ts))

    t_proj = timed(lambda: bsr.w4a4_proj(a, wp, w_sf, s2, out, scratch))
    t_gemm = timed(lambda: bsr.w4a4_gemm(ap, a_sf, as2, wp, w_sf, s2, out, status))
    if int(status.item()) != 0 or bsr.device_status() != 0:
        raise RuntimeError("W4A4 GEMM: a pipeline wait timed out")
    ops = prefill_ops(m, n, k)
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    del wp, w_sf, a, out, scratch, ap, ae, as2, a_sf, flush
    torch.cuda.empty_cache()
    return {"shape": [m, n, k], "tops_proj": ops / t_proj / 1e9, "ms_proj": t_proj,
            "gemm_tops": ops / t_gemm / 1e9, "ms_gemm": t_gemm,
            "fp4_peak": fp4_peak, "gemm_frac_of_fp4_peak": ops / t_gemm / 1e9 / fp4_peak,
            "peak_source": f"measured bf16 burst x {FP4_PER_BF16:g} (nominal dense FP4/bf16 ratio)",
            "static_weight": True,
           "note": "NVFP4 activations and weight; not bit-compatible with the int8 path"}


def stacked_decode_extra(device, steps, peaks, cpu=True):
    """Decode over a stacked weight shaped like Q, K and V of a grouped-query
    layer (4096 + 1024 + 1024 rows, K = 4096, M = 1): one stacked launch per
    step against one launch per segment, each a CUDA-graph loop over
    rotating weight copies (>= 3x L2), static-weight option on."""
    import torch

    import block_scaled_precision_requant_b200 as bsr
    from block_scaled_precision_requant_b200 import synth

    k, ns = 4096, (4096, 1024, 1024)
    a = torch.from_numpy(synth.make_activations(1, k, 1, "normal_outlier_channels")[0].view(np.int16)).view(
        torch.bfloat16).to(device)
    segs = []
    for i, n in enumerate(ns):
        w = synth.make_weight(n, k, 1 + i)
        segs.append(bsr.requant_w(torch.from_numpy(w["w_packed"]).to(device), torch.from_numpy(w["w_e4m3"]).to(device),
                                  float(w["scale2"])))
    nbytes = sum(n * k + n * k // 8 + 2 * n for n in ns) + 2 * k
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(2, -(-3 * l2 // nbytes))
    sets = [[(w.clone(), s.clone()) for w, s in segs] for _ in range(copies)]
    out = torch.empty((1, sum(ns)), dtype=torch.bfloat16, device=device)
    offs = np.cumsum((0,) + ns)

    def stacked(i):
        bsr.decode_stacked(a, sets[i % copies], out, static_weight=True)

    def separate(i):
        for j, (w, s) in enumerate(sets[i % copies]):
            bsr.decode(a, w, s, out[:, offs[j]:offs[j + 1]], static_weight=True)

    res = {}
    for name, fn in (("stacked", stacked), ("separate", separate)):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        res[name] = {"ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9, "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 /
                     peaks["hbm_gbs"]}
        del g
    res["segments"] = list(ns)
    res["bytes_per_step"] = nbytes
    if cpu:
        import oracle

        a_bits = synth.make_activations(1, k, 1, "normal_outlier_channels")[0]
        hw = []
        for i, n in enumerate(ns):
            w = synth.make_weight(n, k, 1 + i)
            hw.append(oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k))
        t, calls = oracle_seconds(lambda: [oracle.proj_rows(a_bits, wq, wsc) for wq, wsc in hw], 3.0)
        res["cpu_baseline"] = {"kind": "oracle", "cores": 1, "gbs": nbytes / t / 1e9, "ms_per_step": t * 1e3,
                               "sample": f"{calls} full step(s) over the three segments (M=1)"}
    del sets
    torch.cuda.empty_cache()
    return res


def w4a16_extra(g, steps, peaks, cpu=True):
    """The NVFP4 W4A16 decode GEMV on the decode workload's weight as stored
    (0.5625 B per weight element): a CUDA-graph loop over rotating copies
    (>= 3x L2), bytes = N*K*0.5625 + 2MK + 2MN per step."""
    torch, bsr = g.torch, g.bsr
    m, n, k = g.wl.shape
    nbytes = n * k // 2 + n * k // 16 + 2 * m * k + 2 * m * n
    l2 = torch.cuda.get_device_properties(g.dev).L2_cache_size
    copies = max(2, -(-3 * l2 // nbytes))
    ws = [(g.wp.clone(), g.we.clone()) for _ in range(copies)]
    s2 = float(g.host["scale2"])
    out = torch.empty((m, n), dtype=torch.bfloat16, device=g.dev)
    for i in range(3):
        bsr.w4a16_decode(g.a, *ws[i % copies], s2, out, static_weight=True)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for i in range(steps):
            bsr.w4a16_decode(g.a, *ws[i % copies], s2, out, static_weight=True)
    gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    gr.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del gr, ws
    g.check_status()
    res = {"ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9, "bytes_per_step": nbytes,
           "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
           "traffic": stored_traffic("nvfp4_gemv_kernel", "decode_w4a16"), "static_weight": True,
           "note": "reads the NVFP4 weight as stored; not bit-compatible with the int8 path"}
    if cpu:
        import oracle

        hd = g.host
        t, calls = oracle_seconds(lambda: oracle.w4a16_gemv(hd["a_bits"], hd["w_packed"], hd["w_e4m3"], hd["scale2"],
                                                            k), 3.0)
        res["cpu_baseline"] = {"kind": "oracle", "cores": 1, "gbs": nbytes / t / 1e9, "ms_per_step": t * 1e3,
                               "sample": f"{calls} full step(s) (M={m})"}
    return res


def oracle_seconds(fn, budget_s, max_calls=50):
    """Mean host seconds of fn() over calls bounded by budget_s."""
    done, spent = 0, 0.0
    while done < 1 or (spent < budget_s and done < max_calls):
        t0 = time.perf_counter()
        fn()
        spent += time.perf_counter() - t0
        done += 1
    return spent / done, done


def w4a4_extra(device, wl, host, steps, peaks, cpu=True):
    """The NVFP4 W4A4 decode GEMV (activation rows quantised to NVFP4 inside
    the kernel) on the decode workload's weight as stored: a CUDA-graph loop
    over rotating copies (>= 3x L2), bytes = N*K*0.5625 + 2MK + 2MN per step."""
    import torch

    import block_scaled_precision_requant_b200 as bsr

    m, n, k = wl.shape
    nbytes = n * k // 2 + n * k // 16 + 2 * m * k + 2 * m * n
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(2, -(-3 * l2 // nbytes))
    wp = torch.from_numpy(host["w_packed"]).to(device)
    we = torch.from_numpy(host["w_e4m3"]).to(device)
    a = torch.from_numpy(host["a_bits"].view(np.int16)).view(torch.bfloat16).to(device)
    ws = [(wp.clone(), we.clone()) for _ in range(copies)]
    s2 = float(host["scale2"])
    out = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    for i in range(3):
        bsr.w4a4_decode(a, *ws[i % copies], s2, out, static_weight=True)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for i in range(steps):
            bsr.w4a4_decode(a, *ws[i % copies], s2, out, static_weight=True)
    gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    gr.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del gr, ws
    if bsr.device_status() != 0:
        raise RuntimeError(f"device status word {bsr.device_status()}")
    res = {"ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9, "bytes_per_step": nbytes,
           "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
           "traffic": stored_traffic("nvfp4_gemv_kernel", "decode_w4a4"), "static_weight": True,
           "note": "NVFP4 activations and weight; not bit-compatible with the int8 path"}
    if cpu:
        import oracle

        t, calls = oracle_seconds(lambda: oracle.w4a4_proj(host["a_bits"], host["w_packed"], host["w_e4m3"],
                                                           host["scale2"], k), 3.0)
        res["cpu_baseline"] = {"kind": "oracle", "cores": 1, "gbs": nbytes / t / 1e9, "ms_per_step": t * 1e3,
                               "sample": f"{calls} full step(s) (M={m})"}
    return res


def stacked_prefill_extra(device, steps, warmup):
    """Prefill over a stacked weight shaped like Q, K and V of a grouped-query
    layer (4096 + 1024 + 1024 rows, K = 4096, M = 2048): bsr_proj_stacked
    (requant_a once, the segments' GEMMs concurrently with grids in
    proportion to their tiles) against one bsr_proj per segment; L2 flushed
    before every step."""
    import torch

    import block_scaled_precision_requant_b200 as bsr
    from block_scaled_precision_requant_b200 import synth

    m, k, ns = 2048, 4096, (4096, 1024, 1024)
    a = torch.from_numpy(synth.make_activations(m, k, 2, "normal_outlier_channels")[0].view(np.int16)).view(
        torch.bfloat16).to(device)
    segs = []
    for i, n in enumerate(ns):
        w = synth.make_weight(n, k, 2 + i)
        segs.append(bsr.requant_w(torch.from_numpy(w["w_packed"]).to(device), torch.from_numpy(w["w_e4m3"]).to(device),
                                  float(w["scale2"])))
    out = torch.empty((m, sum(ns)), dtype=torch.bfloat16, device=device)
    outs = [torch.empty((m, n), dtype=torch.bfloat16, device=device) for n in ns]
    scratch = torch.empty((bsr.proj_scratch_bytes(m, k),), dtype=torch.uint8, device=device)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=device)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.mean(ts))

    t_st = timed(lambda: bsr.proj_stacked(a, segs, out, scratch))
    t_sep = timed(lambda: [bsr.proj(a, w, s, o, scratch) for (w, s), o in zip(segs, outs)])
    ops = 2 * m * sum(ns) * k
    status = bsr.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    del segs, out, outs, scratch, flush
    torch.cuda.empty_cache()
    return {"segments": list(ns), "m": m, "k": k, "stacked": {"ms": t_st, "tops": ops / t_st / 1e9},
            "separate": {"ms": t_sep, "tops": ops / t_sep / 1e9}}


def silu_extra(g, steps, warmup, cpu=True):
    """The down projection from gate/up activations: the fused SiLU.mul
    quantiser + GEMM against the unfused SiLU.mul + requant_a + GEMM."""
    torch, bsr = g.torch, g.bsr
    from block_scaled_precision_requant_b200 import synth

    m, n, k = g.wl.shape
    gb, ub, _ = synth.make_gate_up(m, k, g.wl.seed)
    gate = torch.from_numpy(gb.view(np.int16)).view(torch.bfloat16).to(g.dev)
    up = torch.from_numpy(ub.view(np.int16)).view(torch.bfloat16).to(g.dev)
    cpu_res = None
    if cpu:
        import oracle

        rows = 4
        t, calls = oracle_seconds(lambda: oracle.requant_silu_a(gb[:rows], ub[:rows]), 3.0)
        cpu_res = {"kind": "oracle", "cores": 1, "requant_silu_a_gbs": rows * k * 5.125 / t / 1e9,
                   "sample": f"requant_silu_a of {rows} rows x K={k}, {calls} call(s)"}
    del gb, ub
    x = torch.empty((m, k), dtype=torch.bfloat16, device=g.dev)
    scratch = torch.empty((bsr.proj_silu_scratch_bytes(m, k),), dtype=torch.uint8, device=g.dev)
    t_fused = mean_ms(g.timed(lambda: bsr.proj_silu(gate, up, g.w_i8, g.w_s, g.out, scratch), steps, warmup))
    t_quant = mean_ms(g.timed(lambda: bsr.requant_silu_a(gate, up, g.a_i8, g.a_st), steps, warmup))
    t_mul = mean_ms(g.timed(lambda: bsr.silu_mul(gate, up, x), steps, warmup))
    t_unfused = mean_ms(g.timed(lambda: (bsr.silu_mul(gate, up, x), bsr.proj(x, g.w_i8, g.w_s, g.out, g.scratch)),
                                steps, warmup))
    g.check_status()
    ops = prefill_ops(m, n, k)
    return {
        "tops_fused": ops / t_fused / 1e9,
        "tops_unfused": ops / t_unfused / 1e9,
        "requant_silu_a_gbs": m * k * 5.125 / t_quant / 1e6,
        "silu_mul_gbs": m * k * 6 / t_mul / 1e6,
        "ms": {"proj_silu": t_fused, "silu_mul_then_proj": t_unfused, "requant_silu_a": t_quant, "silu_mul": t_mul},
        "cpu_baseline": cpu_res,
    }


def gpu_main(args):
    import torch

    rank, world, local = dist_init("nccl")
    if not torch.cuda.is_available():
        raise RuntimeError("no CUDA device: the GPU arm has no CPU fallback")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    pci = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    peaks, peak_src = load_peaks()
    extras = not args.no_extra and world == 1
    int8_peak = measure_int8_peak(dev) if extras or args.workload != "decode" else None

    g = Gpu(args.workload, dev)
    wl = g.wl
    m, n, k = wl.shape
    units, unit, metric = units_per_step(wl)
    decode = m <= g.bsr.DECODE_MAX_M

    with ClockSampler(pci) as clk:
        if decode:
            t_steps = g.timed_graph_rotating(args.steps, args.warmup)
        else:
            t_steps = g.timed(g.step, args.steps, args.warmup)
    # decode: the end-to-end loop captured in a CUDA graph (copies inside
    # every step); the eager per-call figure is reported beside it
    t_e2e_eager = g.timed(g.step_e2e, args.steps, args.warmup)
    t_e2e = g.timed_e2e_graph(args.steps, args.warmup) if decode else t_e2e_eager
    if decode:
        t_kernel = t_steps  # the step is one launch of the decode kernel
        kernel = "decode_kernel"
        t_single = g.timed(lambda: g.bsr.decode(g.a, g.w_i8, g.w_s, g.out), args.steps, args.warmup)
    else:
        with ClockSampler(pci) as clk_kernel:
            t_kernel = g.timed_gemm_only(args.steps, args.warmup)
        kernel = "gemm_kernel"
    t_rw = g.timed_requant_w_only(min(args.steps, 20), args.warmup)
    g.check_status()
    w4 = w4a16_extra(g, max(args.steps, 20), peaks, cpu=not args.no_cpu) if decode and extras else None

    ms_step, ms_e2e, ms_kernel, ms_rw, ms_e2e_eager = dist_max(
        [mean_ms(t_steps), mean_ms(t_e2e), mean_ms(t_kernel), mean_ms(t_rw), mean_ms(t_e2e_eager)],
        device="cuda" if world > 1 else "cpu")
    value = world * units / (ms_step / 1e3)
    e2e_value = world * units / (ms_e2e / 1e3)
    if decode:
        rl = roofline("hbm", decode_bytes(m, n, k) / (ms_kernel / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s",
                      stored_traffic(kernel, wl.name))
        rl["peak_source"] = f"{peak_src} HBM copy (MEASURED_PEAKS.json hbm_gbs)"
        rl["single_launch"] = {"ms": mean_ms(t_single),
                               "gbs": decode_bytes(m, n, k) / (mean_ms(t_single) / 1e3) / 1e9,
                               "how": "one eager launch per step, L2 flushed before each (no overlap of steps)"}
    else:
        # the GEMM is bound by the FP32 pipe (the exact rescale), not by the
        # tensor pipe: report against that bound at the sampled clock, and the
        # measured int8 tensor peak beside it
        achieved = prefill_ops(m, n, k) / (ms_kernel / 1e3) / 1e12
        mhz = clk_kernel.summary()["sm_mhz"] or peaks["sm_max_mhz"]
        rl = roofline("alu", achieved, fma_bound_tops(props.multi_processor_count, mhz), "TOPS",
                      stored_traffic(kernel, wl.name))
        rl["tensor_peak"] = int8_peak
        rl["tensor_frac"] = achieved / int8_peak
        rl["tensor_peak_nominal"] = INT8_NOMINAL_TOPS
        rl["peak_source"] = (f"2 FP32 FMAs per element and 32-block at 128 FMA/clk/SM x {props.multi_processor_count} "
                             f"SMs x {mhz:g} MHz (median SM clock sampled during the GEMM timing); tensor_peak: "
                             f"torch._int_mm int8 8192^3 measured in this run")
    rl["kernel"] = kernel

    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded generator; no dataset or trained weights)",
        "config": {**workload_desc(wl, world), "inputs_sha256": input_hashes(g.host)},
        "roofline": rl,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": 2 * m * k, "d2h_bytes_per_step": 2 * m * n,
                "how": ("CUDA graph of the K steps through bsr_decode_host (copy kernel in, decode, copy "
                        "kernel out each step)" if decode else
                        "eager calls per step through bsr_proj_host (row chunks: copy in, requant_a + GEMM, "
                        "copy out, overlapped across chunks)"),
                "eager_value": world * units / (ms_e2e_eager / 1e3),
                "ms_per_step": ms_e2e},
        "gpu_launches": g.launches_per_step() * args.steps,
        "clocks": clk.summary(),
        "int8_peak_tops": int8_peak,
        "requant_w": {"gbs": n * k * 1.6875 / (ms_rw / 1e3) / 1e9, "ms": ms_rw,
                      "frac_of_hbm": n * k * 1.6875 / (ms_rw / 1e3) / 1e9 / peaks["hbm_gbs"]},
    }
    if decode:
        line["l2_rotating_copies"] = getattr(g, "rotating_copies", None)
    host = g.host
    del g
    torch.cuda.empty_cache()
    if extras:
        detail = {}
        for name in ("ffn_up", "ffn_down", "square_ragged"):
            if name != args.workload:
                detail[name] = prefill_extra(name, dev, min(args.steps, 10), min(args.warmup, 3) or 1, peaks,
                                             int8_peak, pci, cpu=not args.no_cpu)
        # flat summary (scalars only) beside the per-workload records
        flat = {}
        for name, r in detail.items():
            flat[f"{name}_tops_incl_requant"] = r["tops_incl_requant"]
            flat[f"{name}_gemm_tops"] = r["roofline"]["achieved"]
            flat[f"{name}_gemm_frac_fp32_bound"] = r["roofline"]["frac"]
            flat[f"{name}_gemm_frac_int8_peak"] = r["roofline"]["tensor_frac"]
            flat[f"{name}_requant_a_gbs"] = r["requant_a"]["gbs"]
            flat[f"{name}_sm_mhz"] = r["clocks"]["sm_mhz"]
            flat[f"{name}_e2e_tops"] = r["e2e"]["value"]
        line["prefill"] = flat
        line["prefill_detail"] = detail
        if w4 is not None:
            line["w4a16_decode"] = w4
        line["stacked_prefill"] = stacked_prefill_extra(dev, min(args.steps, 10), 3)
        try:
            line["w4a4_gemm"] = w4a4_gemm_extra(dev, min(args.steps, 10), 3, peaks)
        except Exception as exc:  # noqa: BLE001 - reported in the line
            line["w4a4_gemm"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        if decode:
            line["stacked_decode"] = stacked_decode_extra(dev, max(args.steps, 20), peaks, cpu=not args.no_cpu)
            try:  # the last GPU work of the run: an error here costs only this entry
                line["w4a4_decode"] = w4a4_extra(dev, wl, host, max(args.steps, 20), peaks, cpu=not args.no_cpu)
            except Exception as exc:  # noqa: BLE001 - reported in the line
                line["w4a4_decode"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_finish()
    return 0


def only_main(args):
    """One operation of the path alone on the workload, K timed launches
    after W warm-up launches (L2 flushed before each): a short, predictable
    launch sequence for profilers.  Prints its time and throughput."""
    import torch

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    g = Gpu(args.workload, dev)
    bsr = g.bsr
    m, n, k = g.wl.shape
    op = args.only
    if op == "decode":
        fn = lambda: bsr.decode(g.a, g.w_i8, g.w_s, g.out)  # noqa: E731
        units, unit = decode_bytes(m, n, k) / 1e9, "GB/s"
    elif op == "proj":
        fn, units, unit = g.step, prefill_ops(m, n, k) / 1e12, "TOPS"
    elif op == "gemm":
        fn = lambda: bsr.gemm(g.a_i8, g.a_st, g.w_i8, g.w_s, g.out)  # noqa: E731
        units, unit = prefill_ops(m, n, k) / 1e12, "TOPS"
    elif op == "requant_a":
        fn = lambda: bsr.requant_a(g.a, g.a_i8, g.a_st)  # noqa: E731
        units, unit = m * k * 3.125 / 1e9, "GB/s"
    elif op == "requant_w":
        fn = lambda: bsr.requant_w(g.wp, g.we, float(g.host["scale2"]), g.w_i8, g.w_s)  # noqa: E731
        units, unit = n * k * 1.6875 / 1e9, "GB/s"
    elif op in ("w4a16", "w4a4_decode"):
        call = bsr.w4a16_decode if op == "w4a16" else bsr.w4a4_decode
        s2 = float(g.host["scale2"])
        fn = lambda: call(g.a, g.wp, g.we, s2, g.out)  # noqa: E731
        units, unit = (n * k // 2 + n * k // 16 + 2 * m * k + 2 * m * n) / 1e9, "GB/s"
    else:
        from block_scaled_precision_requant_b200 import synth

        gb, ub, _ = synth.make_gate_up(m, k, g.wl.seed)
        gate = torch.from_numpy(gb.view(np.int16)).view(torch.bfloat16).to(dev)
        up = torch.from_numpy(ub.view(np.int16)).view(torch.bfloat16).to(dev)
        fn = lambda: bsr.requant_silu_a(gate, up, g.a_i8, g.a_st)  # noqa: E731
        units, unit = m * k * 5.125 / 1e9, "GB/s"
    ms = mean_ms(g.timed(fn, args.steps, args.warmup))
    g.check_status()
    print(json.dumps({"only": op, "workload": g.wl.name, "ms": ms, "value": units / (ms / 1e3), "unit": unit,
                      "steps": args.steps, "warmup": args.warmup}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_main(args)
    if args.only:
        return only_main(args)
    return gpu_main(args)


if __name__ == "__main__":
    sys.exit(main())
