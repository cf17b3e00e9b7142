#!/usr/bin/env python
"""Benchmark of the NVFP4 per-token cast on B200.

One step = one call of nvfp4pt_quantize (zero -> fused row/column amax pass ->
TMA encode pass, with the decayed running-absmax update) over the LLM-sized
activation: bf16 [16384, 8192], N(0,1) with 1% outlier channels x50 (seed 2),
rowwise + columnwise outputs, decay 0.99.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Each rank (one per GPU, torchrun for N > 1) casts its own independent matrix
(replicas: the cast has no exchange step at this scale), so the work per GPU is
fixed as N grows ("weak" scaling). Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain single-threaded C definition)
on bounded row slices of the same matrix: the slow reference arm.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K = 16384, 8192
DECAY = 0.99
FALLBACK_HBM_GBS = 6650.0


def algo_bytes(m: int, k: int) -> int:
    """Compulsory bytes of one cast: bf16 read twice, row and column codes and scales
    written once, amax vectors written once."""
    return 2 * (2 * m * k) + 2 * (m * k // 2) + 2 * (m * k // 16) + 4 * m + 4 * k


def workload_name(m: int, k: int) -> str:
    return f"llm_activation_{m}x{k}_bf16_rowcol_decay0.99"
PROFILE_JSON = os.path.join(ROOT, "profiles", "nvfp4pt_cast_llm_16384x8192.json")
KERNEL_SOURCES = [os.path.join(ROOT, "precision_quantization_row_b200", "csrc", f)
                  for f in ("nvfp4pt_api.cu", "nvfp4pt_device.cuh", "nvfp4pt_kernels.cuh", "nvfp4pt_rowpass.cuh",
                            "nvfp4pt_colpass.cuh", "nvfp4pt_colpass_tma.cuh", "nvfp4pt_dequant.cuh",
                            "nvfp4pt_xform.cuh")]
# The cast's launches on rows of up to 16384 elements, in order (nvfp4pt_timing.h):
# zeroing, the row pass, the column pass.
KERNELS = ("pass0_zero", "rowpass", "colpass")


def kernel_bytes(name: str, m: int, k: int) -> int:
    """Algorithmic bytes of one launch: what the kernel must read and write at least.
    Row pass: x once; row codes, row scales, row amax; the column amax vector.
    Column pass: x once and the column amax; column codes and scales."""
    if name == "rowpass":
        return 2 * m * k + m * k // 2 + m * k // 16 + 4 * m + 4 * k
    if name == "colpass":
        return 2 * m * k + 4 * k + m * k // 2 + m * k // 16
    return 4 * k


def strip_comments(src: str) -> str:
    """C/C++ source without comments and blank space, so that the hash below changes
    with the code only (string literals here hold no comment markers)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_sha(texts=None) -> str:
    """Hash of the kernel sources' code (comments and spacing do not count)."""
    h = hashlib.sha256()
    if texts is None:
        texts = []
        for p in KERNEL_SOURCES:
            with open(p, encoding="utf-8") as f:
                texts.append(f.read())
    for t in texts:
        h.update(strip_comments(t).encode())
    return h.hexdigest()[:16]


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu summary,
    if it was taken on the current kernel sources (else None)."""
    try:
        with open(PROFILE_JSON) as f:
            d = json.load(f)
        if d.get("kernel_source_sha") == kernel_source_sha():
            return d["kernels"][kernel]["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


# ------------------------------------------------------------- distributed

class Dist:
    """Rank bookkeeping. N = 1 runs without a process group."""

    def __init__(self, gpus: int, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != gpus:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={self.world}")
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            backend = backend or "nccl"
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            if self.pg.get_backend() == "nccl":
                import torch
                self.pg.barrier(device_ids=[torch.cuda.current_device()])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        dev = "cuda" if self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def timed_region(dist: Dist, run, sync) -> float:
    """Barrier + sync on both sides of `run`; returns the max over ranks of the
    seconds `run` reports (device time)."""
    dist.barrier()
    sync()
    secs = run()
    sync()
    dist.barrier()
    return dist.max(secs)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""
    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return
        self.period = period
        self._t = threading.Thread(target=self._loop, daemon=True)

    def _loop(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}



# ------------------------------------------------------- timing + baselines

def repeat_count(args, per_region_s: float) -> int:
    """Timed regions of `steps` steps each: --repeats, else enough for ~1 s of timed work
    (at least 5, at most 50), so that the median is steady and NVML sees many samples."""
    if args.repeats > 0:
        return args.repeats
    return int(max(5, min(50, 1.0 / max(per_region_s, 1e-6))))


def timed_regions(args, dist: Dist, dev, stream, step) -> tuple[float, list, dict]:
    """Warm-up, then R timed regions of `args.steps` steps each (CUDA events on the
    launching stream, barrier + sync on both sides, max over ranks), NVML sampled over
    all of them. Returns (median region seconds, all region seconds, clock summary)."""
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def region():
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        ev1.synchronize()
        return ev0.elapsed_time(ev1) / 1e3

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    probe = timed_region(dist, region, lambda: torch.cuda.synchronize(dev))
    reps = repeat_count(args, probe)
    secs = []
    with ClockSampler(dev.index) as clk:
        for _ in range(reps):
            secs.append(timed_region(dist, region, lambda: torch.cuda.synchronize(dev)))
    return statistics.median(secs), secs, clk.summary()


def region_stats(secs: list) -> dict:
    ms = sorted(s * 1e3 for s in secs)
    return {"repeats": len(ms), "region_ms_min": ms[0], "region_ms_median": statistics.median(ms),
            "region_ms_max": ms[-1]}


def cpu_info() -> dict:
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def pinned(fn):
    """Run fn() with this process pinned to one core (the first it may use), as
    `taskset -c <core>` would; returns (fn's result, seconds, core)."""
    old = os.sched_getaffinity(0)
    core = min(old)
    os.sched_setaffinity(0, {core})
    try:
        t = time.perf_counter()
        r = fn()
        return r, time.perf_counter() - t, core
    finally:
        os.sched_setaffinity(0, old)


def oracle_baseline(elems: int, run, sample: str, unit_scale=None) -> dict:
    """The oracle as it stands, single-threaded, pinned to one core, on a bounded sample:
    `run()` does `elems` elements of the workload's cast."""
    _, secs, core = pinned(run)
    d = {"value": elems / secs, "unit": "elem/s", "cores": 1, "kind": "oracle", "sample": sample,
         "seconds": secs, "pinned_core": core}
    d.update(cpu_info())
    return d


# --------------------------------------------------------------- GPU arm

def run_gpu(args, dist: Dist) -> dict | None:
    global M, K
    M, K = args.rows, args.cols
    import torch

    import precision_quantization_row_b200 as nv
    from precision_quantization_row_b200 import build, inputs

    build.build()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream(dev)

    x_host = inputs.llm(M=M, K=K)  # same matrix on every rank: independent replicas
    # two input copies and two output sets, rotated every step (all > L2 in total)
    xs = [x_host.to(dev), x_host.to(dev).clone()]
    outs = [nv._outputs(M, K, nv.ROWWISE | nv.COLWISE, dev) for _ in range(2)]
    buf = torch.zeros(1, dtype=torch.float32, device=dev)
    ws = nv.new_workspace(M, K, device=dev)

    def step(i):
        nv.quantize(xs[i & 1], absmax=buf, decay=DECAY, out=outs[i & 1], workspace=ws, stream=stream)

    secs, all_secs, clocks = timed_regions(args, dist, dev, stream, step)
    if nv.workspace_error(ws) != 0:
        raise RuntimeError("device error word set during the timed region")
    launches = nv.CAST_LAUNCHES * args.steps  # zero, row pass, column pass per cast

    # Per-kernel times: the same casts through the timed entry, which records an event
    # before the first launch and after each launch on the casts' stream.
    kt_steps = min(args.steps, 200)
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(nv.CAST_LAUNCHES + 1)] for _ in range(kt_steps)]
    for row in kevs:
        for e in row:
            e.record(stream)

    def run_kernels():
        for i in range(kt_steps):
            nv.quantize_timed(xs[i & 1], kevs[i], absmax=buf, decay=DECAY, out=outs[i & 1], workspace=ws,
                              stream=stream)
        kevs[-1][-1].synchronize()
        return 0.0

    timed_region(dist, run_kernels, lambda: torch.cuda.synchronize(dev))
    kernel_ms = {name: dist.max(sum(row[j].elapsed_time(row[j + 1]) for row in kevs) / kt_steps)
                 for j, name in enumerate(KERNELS)}

    e2e = None if args.no_e2e else run_e2e(args, dist, dev, stream, x_host, xs, outs, buf, ws)
    if nv.workspace_error(ws) != 0:
        raise RuntimeError("device error word set during the timed region")

    if dist.rank != 0:
        return None
    peak, peak_kind = measured_peak()
    per_cast = secs / args.steps
    cast_achieved = algo_bytes(M, K) / per_cast / 1e9
    dominant = max(("rowpass", "colpass"), key=lambda n: kernel_ms[n])
    achieved = kernel_bytes(dominant, M, K) / (kernel_ms[dominant] / 1e3) / 1e9
    traffic = ncu_traffic(dominant)
    elems = float(M) * K
    line = {
        "metric": "NVFP4 per-token cast: elems/s, achieved HBM GB/s, % of B200 HBM peak",
        "value": elems * args.steps * dist.world / secs,
        "unit": "elem/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": per_cast * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16->nvfp4 (e2m1 codes, e4m3 scales, fp32 amax)",
        "data": "synthetic",
        "config": {"workload": workload_name(M, K), "rows": M, "cols": K, "flags": "rowwise+columnwise",
                   "absmax_decay": DECAY, "parallelism": f"replicas x{dist.world}",
                   "l2": f"inputs larger than L2 ({M * K * 2 / 1e6:.0f} MB each), 2 rotating input copies "
                         "and output sets"},
        "timing": dict(region_stats(all_secs), note="value and ms_per_step: the median region"),
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": kernel_bytes(dominant, M, K),
                     "launch_us": kernel_ms[dominant] * 1e3,
                     "kernels_us": {n: round(v * 1e3, 2) for n, v in kernel_ms.items()},
                     "kernels_note": f"CUDA events around each launch, {kt_steps} casts; the launches "
                                     "then run one after another",
                     "cast": {"achieved": cast_achieved, "frac": cast_achieved / peak,
                              "nominal_frac_8TBs": cast_achieved / 8000.0,
                              "algorithmic_bytes_per_cast": algo_bytes(M, K)}},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return line


def run_e2e(args, dist: Dist, dev, stream, x_host, xs, outs, buf, ws) -> dict:
    """The public call end to end with host buffers: every step copies its input from
    pinned host memory and every output (codes, scales, amax vectors, buffer) back. The
    copies run on their own streams, two buffer sets deep, so that step i+1's input
    crosses PCIe while step i's outputs come back (full duplex); the timed region runs
    from the first copy in to the last copy out."""
    import torch

    import precision_quantization_row_b200 as nv
    m, k = x_host.shape
    xh = x_host.pin_memory()
    host_out = [{n: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for n, v in outs[0].items()}
                for _ in range(2)]
    buf_h = [torch.empty(1, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    h2d = xh.numel() * xh.element_size()
    d2h = sum(v.numel() * v.element_size() for v in host_out[0].values()) + 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = max(4, min(args.steps, 12))
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_c = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def region():
        t0.record(s_in)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_c[i - 2])       # the cast of step i-2 has read xs[b]
            with torch.cuda.stream(s_in):
                xs[b].copy_(xh, non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])   # step i-2's outputs have left outs[b]
            nv.quantize(xs[b], absmax=buf, decay=DECAY, out=outs[b], workspace=ws, stream=stream)
            ev_c[i].record(stream)
            s_out.wait_event(ev_c[i])
            with torch.cuda.stream(s_out):
                for name, v in outs[b].items():
                    host_out[b][name].copy_(v, non_blocking=True)
                buf_h[b].copy_(buf, non_blocking=True)
            ev_out[i].record(s_out)
        s_out.wait_event(ev_c[n - 1])
        t1.record(s_out)
        t1.synchronize()
        return t0.elapsed_time(t1) / 1e3

    timed_region(dist, region, lambda: torch.cuda.synchronize(dev))   # warm-up of the copy path
    secs = statistics.median(timed_region(dist, region, lambda: torch.cuda.synchronize(dev)) for _ in range(3))
    return {"value": float(m) * k * n * dist.world / secs, "unit": "elem/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "note": "pinned host buffers; copy-in, cast and copy-out on three streams, two buffer sets deep"}


def op_bytes(op: str, m: int, k: int) -> int:
    """Algorithmic bytes of the secondary ops. Dequantize: rowwise codes, scales and
    amax in, bf16 out. Columnwise requantize: rowwise data in, columnwise data out
    (the least any implementation must move)."""
    rowdata = m * k // 2 + m * k // 16 + 4 * m
    if op == "dequant":
        return rowdata + 2 * m * k
    return rowdata + m * k // 2 + m * k // 16 + 4 * k


def run_gpu_op(args, dist: Dist, op: str) -> dict | None:
    """Device time of nvfp4pt_dequantize or nvfp4pt_requantize_colwise on the rowwise
    outputs of the headline activation (two rotating input sets)."""
    import torch

    import precision_quantization_row_b200 as nv
    from precision_quantization_row_b200 import build, inputs

    build.build()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream(dev)
    m, k = args.rows, args.cols
    x = inputs.llm(M=m, K=k).to(dev)
    srcs = [nv.quantize(x, flags=nv.ROWWISE), nv.quantize(x.neg(), flags=nv.ROWWISE)]
    del x
    if op == "dequant":
        outs = [torch.empty((m, k), dtype=torch.bfloat16, device=dev) for _ in range(2)]

        def step(i):
            s = srcs[i & 1]
            nv.dequantize(s["q_row"], s["sf_row"], s["amax_row"], out=outs[i & 1], stream=stream)
        launches = 1
    else:
        ws = torch.empty(nv.requantize_workspace_bytes(m, k, 1), dtype=torch.uint8, device=dev)
        outs = [None, None]

        def step(i):
            s = srcs[i & 1]
            outs[i & 1] = nv.requantize_colwise(s["q_row"], s["sf_row"], s["amax_row"], out=outs[i & 1],
                                                workspace=ws, stream=stream)
        # rows up to 16384 wide: the cast's three kernels read the NVFP4 data directly;
        # wider: a dequantize launch first
        launches = nv.CAST_LAUNCHES + (0 if k <= 16384 else 1)
    secs, all_secs, clocks = timed_regions(args, dist, dev, stream, step)
    if dist.rank != 0:
        return None
    peak, peak_kind = measured_peak()
    per = secs / args.steps
    achieved = op_bytes(op, m, k) / per / 1e9
    name = {"dequant": "NVFP4 rowwise dequantize to bf16", "requant": "NVFP4 rowwise -> columnwise requantize"}[op]
    return {
        "metric": f"{name}: elems/s, achieved HBM GB/s", "value": float(m) * k * args.steps * dist.world / secs,
        "unit": "elem/s", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4->bf16" if op == "dequant" else "nvfp4->nvfp4 (bf16 values in registers)", "data": "synthetic",
        "config": {"workload": f"{op}_rowwise_{m}x{k}", "rows": m, "cols": k,
                   "l2": "two rotating input sets and outputs"},
        "timing": region_stats(all_secs),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_kind, "algorithmic_bytes_per_call": op_bytes(op, m, k)},
        "gpu_launches": launches * args.steps, "clocks": clocks,
    }


def run_gpu_opts(args, dist: Dist) -> dict | None:
    """Device time of nvfp4pt_quantize_grouped_opts (one token group) on the headline
    activation with the columnwise options: rht (the 16-point transform; its own amax
    sweep reads x a third time), sr (stochastic rounding, Philox words) or rht_sr."""
    import torch

    import precision_quantization_row_b200 as nv
    from precision_quantization_row_b200 import build, inputs

    build.build()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream(dev)
    m, k = args.rows, args.cols
    x_host = inputs.llm(M=m, K=k)
    xs = [x_host.to(dev), x_host.to(dev).clone()]
    outs = [nv._outputs(m, k, nv.ROWWISE | nv.COLWISE, dev) for _ in range(2)]
    buf = torch.zeros(1, dtype=torch.float32, device=dev)
    ws = nv.new_workspace(m, k, device=dev)
    mode = args.colwise_opts
    opts = dict(rht="rht" in mode, rht_signs=0xB65C if "rht" in mode else 0, sr="sr" in mode, seed=2024)

    def step(i):
        nv.quantize_grouped_opts(xs[i & 1], None, absmax=buf, decay=DECAY, out=outs[i & 1], workspace=ws,
                                 stream=stream, offset=i, **opts)

    secs, all_secs, clocks = timed_regions(args, dist, dev, stream, step)
    if nv.workspace_error(ws) != 0:
        raise RuntimeError("device error word set during the timed region")
    if dist.rank != 0:
        return None
    peak, peak_kind = measured_peak()
    per = secs / args.steps
    byts = algo_bytes(m, k) + (2 * m * k if opts["rht"] else 0)   # the transform's amax sweep reads x again
    achieved = byts / per / 1e9
    return {
        "metric": "NVFP4 per-token cast with columnwise options: elems/s, achieved HBM GB/s",
        "value": float(m) * k * args.steps * dist.world / secs, "unit": "elem/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->nvfp4", "data": "synthetic",
        "config": {"workload": f"{workload_name(m, k)}_colwise_{mode}", "rows": m, "cols": k,
                   "l2": "inputs larger than L2, 2 rotating input copies and output sets"},
        "timing": region_stats(all_secs),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_kind, "algorithmic_bytes_per_call": byts},
        "gpu_launches": (nv.CAST_LAUNCHES + (1 if opts["rht"] else 0)) * args.steps, "clocks": clocks,
    }


def measured_tensor_peak():
    """Dense FP4 tensor peak: the measured bf16 burst (cuBLAS) times the nominal FP4/bf16
    ratio 4 (9 and 2.25 PFLOP/s dense), or the fallback bf16 figure times 4."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 4 (nominal fp4/bf16)"
    except Exception:
        return 4.0 * 1590.0, "fallback bf16 x 4 (nominal fp4/bf16)"


def run_gpu_gemm(args, dist: Dist) -> dict | None:
    """Device time of nvfp4pt_gemm_per_token on the forward product of the headline layer:
    A = the rowwise cast of the 16384 x 8192 activation, B = the rowwise cast of an
    8192 x 8192 weight (N(0, 0.02)), D = A B^T in fp32 (two output buffers rotate)."""
    import torch

    import precision_quantization_row_b200 as nv
    from precision_quantization_row_b200 import build, inputs

    build.build()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream(dev)
    m, k, n = args.rows, args.cols, args.gemm_n
    x = inputs.llm(M=m, K=k).to(dev)
    g = torch.Generator(device=dev).manual_seed(6)
    w = (torch.randn((n, k), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    a = nv.quantize(x, flags=nv.ROWWISE)
    b = nv.quantize(w, flags=nv.ROWWISE)
    del x, w
    outs = [torch.empty((m, n), dtype=torch.float32, device=dev) for _ in range(2)]
    ws = nv.new_gemm_workspace(m, n, k, dev)

    def step(i):
        nv.gemm_per_token(a["q_row"], a["sf_row"], a["amax_row"], b["q_row"], b["sf_row"], b["amax_row"],
                          out=outs[i & 1], workspace=ws, stream=stream)

    secs, all_secs, clocks = timed_regions(args, dist, dev, stream, step)
    if nv.workspace_error(ws) != 0:
        raise RuntimeError("device error word set during the timed region")
    if dist.rank != 0:
        return None
    peak, peak_kind = measured_tensor_peak()
    per = secs / args.steps
    flops = 2.0 * m * n * k
    tflops = flops / per / 1e12
    line = {
        "metric": "NVFP4 per-token GEMM (block-scaled tcgen05, amax-vector epilogue): TFLOP/s",
        "value": flops * args.steps * dist.world / secs / 1e12, "unit": "TFLOP/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 x nvfp4 -> fp32 (e2m1, e4m3 block16 scales)",
        "data": "synthetic",
        "config": {"workload": f"gemm_fprop_{m}x{n}x{k}", "m": m, "n": n, "k": k,
                   "l2": "operands 151 MB, 2 rotating fp32 outputs of " f"{m * n * 4 / 1e6:.0f} MB"},
        "timing": region_stats(all_secs),
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None, "peak_source": peak_kind,
                     "algorithmic_flops_per_call": flops},
        "gpu_launches": args.steps, "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cpu = lambda t: t.cpu().numpy()
        rows = 32
        A = [cpu(a[n_][:rows]) for n_ in ("q_row", "sf_row", "amax_row")]
        B = [cpu(b[n_][:rows]) for n_ in ("q_row", "sf_row", "amax_row")]
        base = oracle_baseline(0, lambda: oracle.gemm_per_token(*A, *B),
                               f"the exact-sum oracle on the first {rows} rows of A x the first {rows} rows of B "
                               f"(k = {k})")
        base["value"] = 2.0 * rows * rows * k / base["seconds"] / 1e12
        base["unit"] = "TFLOP/s"
        line["cpu_baseline"] = base
    return line


def run_gpu_config(args, dist: Dist, config: str) -> dict | None:
    """Device time per call of the other workloads (parity-test configurations, reported
    beside the headline): dense 4096x4096 row+column cast, the grouped MoE cast
    (65536x7168, 64 token groups), the 16x16 weight cast (28672x8192) and the calibration
    stream (200 activations of 8192x4096 through the fused cast and the decayed buffer at
    decay 0.99; one step = one activation). Two input copies rotate (the dense one fits
    L2: 8 copies rotate there; the stream's 200 activations are all distinct)."""
    import torch

    import precision_quantization_row_b200 as nv
    from precision_quantization_row_b200 import build, inputs

    build.build()
    torch.cuda.set_device(dist.local_rank)
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream(dev)
    offsets = None
    if config == "dense":
        x = inputs.dense().to(dev)
        m, k, g, copies = x.shape[0], x.shape[1], 1, 8
    elif config == "moe":
        xh, offsets = inputs.moe()
        x = xh.to(dev)
        m, k, g, copies = x.shape[0], x.shape[1], len(offsets) - 1, 2
    elif config == "weight":
        x = inputs.weight().to(dev)
        m, k, g, copies = x.shape[0], x.shape[1], 1, 2
    else:   # calib
        m, k, g, copies = 8192, 4096, 1, 200
        x = None
    if config == "calib":
        xs = [inputs.calib_step(t, m, k, device=str(dev)) for t in range(copies)]
    else:
        xs = [x] + [x.clone() for _ in range(copies - 1)]
    ws = nv.new_workspace(m, k, g, device=dev)
    if config == "moe":
        outs = [None] * copies
        bufs = torch.zeros(g, dtype=torch.float32, device=dev)

        def step(i):
            outs[i % copies] = nv.quantize_grouped(xs[i % copies], offsets, absmax=bufs, decay=DECAY,
                                                   out=outs[i % copies], workspace=ws, stream=stream)
        byts = 2 * (2 * m * k) + 2 * (m * k // 2) + 2 * (m * k // 16) + 4 * m + 4 * g * k
    elif config in ("dense", "calib"):
        nout = 2 if config == "calib" else copies
        outs = [nv._outputs(m, k, nv.ROWWISE | nv.COLWISE, dev) for _ in range(nout)]
        buf = torch.zeros(1, dtype=torch.float32, device=dev)

        def step(i):
            nv.quantize(xs[i % copies], absmax=buf, decay=DECAY, out=outs[i % nout], workspace=ws, stream=stream)
        byts = algo_bytes(m, k)
    else:
        outs = [None] * copies

        def step(i):
            outs[i % copies] = nv.quantize_weight_2d(xs[i % copies], out=outs[i % copies], workspace=ws,
                                                     stream=stream)
        # the weight once (a band's second read comes from L2), rowwise outputs
        byts = 2 * m * k + m * k // 2 + m * k // 16 + 4 * m
    if config == "calib":
        args.steps = copies   # one step per activation of the stream
    secs, all_secs, clocks = timed_regions(args, dist, dev, stream, step)
    if nv.workspace_error(ws) != 0:
        raise RuntimeError("device error word set during the timed region")
    if dist.rank != 0:
        return None
    peak, peak_kind = measured_peak()
    per = secs / args.steps
    achieved = byts / per / 1e9
    workload = {"dense": "dense_4096x4096_rowcol", "moe": "moe_grouped_65536x7168_g64_rowcol",
                "weight": "weight_2d_28672x8192", "calib": "calibration_stream_200x8192x4096_decay0.99"}[config]
    line = {
        "metric": "NVFP4 per-token cast: elems/s, achieved HBM GB/s, % of B200 HBM peak",
        "value": float(m) * k * args.steps * dist.world / secs, "unit": "elem/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->nvfp4", "data": "synthetic",
        "config": {"workload": workload, "rows": m, "cols": k, "groups": g,
                   "l2": f"{copies} rotating input copies" if config != "calib" else
                         "200 distinct activations (the stream), 2 output sets"},
        "timing": region_stats(all_secs),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "nominal_frac_8TBs": achieved / 8000.0, "traffic": None, "peak_source": peak_kind,
                     "algorithmic_bytes_per_call": byts},
        "gpu_launches": nv.CAST_LAUNCHES * args.steps, "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = config_oracle_baseline(config, xs, offsets, m, k)
    return line


def config_oracle_baseline(config: str, xs, offsets, m: int, k: int) -> dict:
    """The oracle on a bounded sample of the workload, pinned to one core."""
    import numpy as np

    import oracle
    oracle.build()
    if config == "calib":
        # steps t = 0, 99 and 199 of the stream, each a full cast with the buffer update
        ts = (0, 99, 199)
        samples = [oracle._bits(xs[t].cpu()) for t in ts]

        def run():
            buf = 0.0
            for s in samples:
                buf = oracle.quantize(s, absmax=buf, decay=DECAY)["absmax"]
        return oracle_baseline(len(ts) * m * k, run, "steps t = 0, 99, 199 of the stream (full casts and "
                               "buffer updates); value = elem/s over the three")
    if config == "moe":
        # the first sixteen token groups, one grouped cast (about 10 s of one core)
        g4 = 16
        rows = int(offsets[g4])
        xb = oracle._bits(xs[0][:rows].cpu())
        off = np.asarray(offsets[:g4 + 1], np.int64)
        return oracle_baseline(rows * k, lambda: oracle.quantize_grouped(xb, off),
                               f"the first {g4} token groups ({rows} rows) as one grouped cast")
    if config == "weight":
        rows = 28672   # the whole weight (about 7 s of one core)
        wb = oracle._bits(xs[0][:rows].cpu())
        return oracle_baseline(rows * k, lambda: oracle.quantize_weight_2d(wb),
                               f"rows 0..{rows - 1} of the weight (2D cast)")
    xb = oracle._bits(xs[0].cpu())   # dense: the whole matrix, five times (about 10 s of one core)

    def run_dense():
        buf = 0.0
        for _ in range(5):
            buf = oracle.quantize(xb, absmax=buf, decay=DECAY)["absmax"]
    return oracle_baseline(5 * m * k, run_dense,
                           f"the whole {m}x{k} matrix five times, full row+col cast with the buffer update")


def headline_oracle_baseline(rows: int) -> dict:
    """The oracle's full row+col cast (with the absmax update) of the first `rows` rows of
    the benchmark matrix, single-threaded and pinned to one core."""
    import oracle
    from precision_quantization_row_b200 import inputs
    oracle.build()
    xb = oracle._bits(inputs.llm()[:rows].contiguous())
    return oracle_baseline(rows * K, lambda: oracle.quantize(xb, absmax=0.0, decay=DECAY),
                           f"rows 0..{rows - 1} of the {M}x{K} matrix ({rows * K} elements), full row+col cast")


def run_reference(args, rank: int, world: int) -> dict | None:
    """The oracle as it stands, single-threaded and pinned to one core, on bounded row
    slices of the same matrix; the slice is sized so that warm-up + timed steps take
    about two minutes."""
    if rank != 0:
        return None
    import oracle
    from precision_quantization_row_b200 import inputs
    oracle.build()
    x = inputs.llm()
    probe = oracle._bits(x[:16].contiguous())
    t = time.perf_counter()
    oracle.quantize(probe, absmax=0.0, decay=DECAY)
    per_row = (time.perf_counter() - t) / 16
    rows = int(120.0 / max(1, args.steps + args.warmup) / max(per_row, 1e-9)) // 16 * 16
    rows = max(16, min(1024, rows))
    samples = [oracle._bits(x[(i * rows) % M:(i * rows) % M + rows].contiguous()) for i in range(4)]

    def run():
        for i in range(args.warmup):
            oracle.quantize(samples[i % 4], absmax=0.0, decay=DECAY)
        t = time.perf_counter()
        for i in range(args.steps):
            oracle.quantize(samples[i % 4], absmax=0.0, decay=DECAY)
        return time.perf_counter() - t

    secs, _, core = pinned(run)
    value = rows * K * args.steps / secs
    base = {"value": value, "unit": "elem/s", "cores": 1, "kind": "oracle", "pinned_core": core,
            "sample": f"{rows}-row slices ({rows * K} elements) of the {M}x{K} matrix per step"}
    base.update(cpu_info())
    return {
        "impl": "reference",
        "metric": "NVFP4 per-token cast: elems/s, achieved HBM GB/s, % of B200 HBM peak",
        "value": value, "unit": "elem/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->nvfp4 (e2m1 codes, e4m3 scales, fp32 amax)", "data": "synthetic",
        "config": {"workload": workload_name(M, K), "rows": M, "cols": K, "flags": "rowwise+columnwise",
                   "absmax_decay": DECAY, "parallelism": "single CPU thread"},
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "elem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--repeats", type=int, default=0,
                    help="timed regions of --steps steps (0: enough for about a second, 5..50)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rows", type=int, default=16384, help="rows of the activation (profiling runs)")
    ap.add_argument("--cols", type=int, default=8192, help="columns of the activation (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--op", choices=["cast", "dequant", "requant", "gemm"], default="cast",
                    help="cast: the per-token cast (the headline); dequant / requant / gemm: the secondary ops")
    ap.add_argument("--gemm-n", type=int, default=8192, help="N of --op gemm (M = --rows, K = --cols)")
    ap.add_argument("--colwise-opts", choices=["rht", "sr", "rht_sr"], default=None,
                    help="time the cast with these columnwise options (the headline activation)")
    ap.add_argument("--config", choices=["llm", "dense", "moe", "weight", "calib"], default="llm",
                    help="llm: the headline activation; the others time the remaining workloads")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        line = run_reference(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dist = Dist(args.gpus)
    try:
        if args.config != "llm":
            line = run_gpu_config(args, dist, args.config)
        elif args.colwise_opts:
            line = run_gpu_opts(args, dist)
        elif args.op == "gemm":
            line = run_gpu_gemm(args, dist)
        elif args.op != "cast":
            line = run_gpu_op(args, dist, args.op)
        else:
            line = run_gpu(args, dist)
            if line is not None and dist.world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = headline_oracle_baseline(12288)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
