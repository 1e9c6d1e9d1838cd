#!/usr/bin/env python
"""Benchmark of the weight-only quantized projection GEMM on B200.

Default workload ("blocks12_m4096"): the 12 RT-J blocks' mixed q4/q8
projection sets resident on the GPU (qkvg q4 2048x512, wo q8 512x512, w13 q4
4096x512, w2 q8 512x2048 per block, independent seeds), run back to back at
M = 4096 activation rows (B=4, S=1024 cells) through rt_qblock_project.  One
step = the 12 blocks' 48 projections over one batch.  Inputs and outputs
together stream ~2 GB per step, more than L2, so no flush is needed.

Printed as one JSON line (rank 0):
  value      whole-job TFLOP/s (2*M*N*K summed over the step's projections),
             device-timed with CUDA events, max over ranks; the step's calls
             are captured once as a CUDA graph and replayed (config.issue;
             --eager issues them call by call);
  e2e        the same metric with the step's inputs copied from pinned host
             memory and its outputs copied back inside the timed region (with
             whole blocks, block by block on two copy streams beside the
             compute stream, as a caller of the block driver would);
  roofline   the dominant call of the step (the projection, or the block's
             projections that share one launch of the activation-resident
             kernel, with the largest share of the step), its algorithmic
             bytes or flops over its CUDA-event duration, against
             MEASURED_PEAKS.json;
  cpu_baseline  the CPU oracle on a bounded row sample of the same workload.

`--impl reference` times the CPU oracle itself (rank 0 only) on the same
workload, metric and unit, one bounded row sample per step.

Other workloads (`--workload`), each printing one line of the same form:
  block_m80, block_m2048, block_m4096
               one block's projection set at M = 80 (one grouped launch; the
               roofline object then describes that launch), at M = 2048 and at
               M = 4096 (the default workload's first block, for profiler
               captures).
  rot_m80      small M as an aggregate weight stream: the 12 blocks' weights in
               rotating device copies totalling ~4x L2, every copy's projection
               set at M = 80, 16 copies (64 projections) per rt_qgemm_batch
               call, the step's calls replayed from a CUDA graph; value in GB/s
               of quantized weights.
  m_sweep      M in {1, 2, 4, 8, 16, 32, 80, 512, 4096, 65536} for the q4
               512->2048 and q8 2048->512 shapes on the SIMT path, the
               tensor-core path and RT_PATH_AUTO; value = TFLOP/s of the q4
               shape at M = 65536, every point under `sweep`, the measured
               crossover under `crossover`.
  w13_m4096, w2_m4096, qkvg_m4096, w13_m16384, w2_m16384
               single projections, sized for profiler captures.
  blocks12_q8_m4096, block_q8_m80
               the all-int8 recipe of the int8 card (every projection q8,
               fused qkvg and w13 included) on the 12 blocks at M = 4096 and
               on one block at M = 80 (rt_qblock_project_fmt).

Multi-GPU (torchrun): every rank runs the same step on its own batch (replica
weights, rank-seeded activations, no data-path collective) -> weak scaling.
"""
from __future__ import annotations

import argparse
import math
import ctypes
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from int8_dequant_gemm_b200 import workloads as wl  # noqa: E402

METRIC = "q4/q8 dequant-GEMM GB/s (small M) and TFLOP/s (large M), % roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}

WORKLOADS = {
    # name: (config id for seeds, number of blocks, M, projections)
    "blocks12_m4096": (4, 12, 4096, ("qkvg", "wo", "w13", "w2")),
    "block_m80": (3, 1, 80, ("qkvg", "wo", "w13", "w2")),
    "block_m2048": (3, 1, 2048, ("qkvg", "wo", "w13", "w2")),
    # one block of the default workload (175 MB of inputs and outputs, more
    # than L2), sized for profiler captures of the block's grouped launch
    "block_m4096": (4, 1, 4096, ("qkvg", "wo", "w13", "w2")),
    # single-projection cases sized for profiler captures
    "w13_m4096": (4, 1, 4096, ("w13",)),
    "w2_m4096": (4, 1, 4096, ("w2",)),
    "qkvg_m4096": (4, 1, 4096, ("qkvg",)),
    # small M as an aggregate weight stream (see run_small_m)
    "rot_m80": (4, 0, 80, ("qkvg", "wo", "w13", "w2")),
    # M in {1, 16, 80, 512, 4096, 65536} for the q4 512->2048 and q8 2048->512 shapes
    "m_sweep": (5, 0, 0, ()),
    # outputs larger than L2, for full profiler captures of one launch
    "w13_m16384": (4, 1, 16384, ("w13",)),
    "w2_m16384": (4, 1, 16384, ("w2",)),
    # the int8 card's all-int8 recipe: every projection q8 (fused qkvg and w13 too)
    "blocks12_q8_m4096": (4, 12, 4096, ("qkvg", "wo", "w13", "w2")),
    "block_q8_m80": (3, 1, 80, ("qkvg", "wo", "w13", "w2")),
}

# Workloads that store every projection in one format instead of the mixed
# recipe; proj_dims reports the format in force for this process's workload.
ALL_FORMAT = {"blocks12_q8_m4096": "q8", "block_q8_m80": "q8"}
FORMAT_OVERRIDE = {}


def proj_dims(name):
    spec = wl.BLOCK_PROJECTIONS[name]
    return FORMAT_OVERRIDE.get(name, spec["fmt"]), spec["N"], spec["K"]


def weight_bytes(name):
    fmt, N, K = proj_dims(name)
    return N * K // 2 + N * (K // 32) * 4 if fmt == "q4" else N * K + N * 4


def proj_flops(name, M):
    _, N, K = proj_dims(name)
    return 2 * M * N * K


def proj_bytes(name, M):
    """Algorithmic HBM bytes of one launch: packed weights + fp32 X + fp32 Y."""
    _, N, K = proj_dims(name)
    return weight_bytes(name) + 4 * M * K + 4 * M * N


# ---------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS)


def source_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_dequant_gemm_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (same digest); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    digest = source_digest()
    for line in open(p):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel_key:
            if parts[2] == digest:
                return float(parts[1])
    return None


class NvmlClockSampler:
    """NVML sampling (read-only) of SM clock, power and throttle reasons every
    ~2 ms during a window: the timed regions are milliseconds long, shorter
    than nvidia-smi's sampling period."""
    REASONS = (("hw_slowdown", "nvmlClocksThrottleReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksThrottleReasonSwPowerCap", 0x4))

    def __init__(self, gpu_id):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        if isinstance(gpu_id, str) and gpu_id.startswith("GPU-"):
            self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_id)
        else:
            self.h = pynvml.nvmlDeviceGetHandleByIndex(int(gpu_id))
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.masks = [(n, getattr(pynvml, a, d)) for n, a, d in self.REASONS]
        self.samples = []
        self.running = False

    def start(self):
        self.running = True
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def _loop(self):
        nv = self.nv
        while self.running:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                why = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                watts = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((time.time(), mhz, why, watts))
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self):
        self.running = False
        self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [r for r in self.samples if t0 <= r[0] <= t1] or self.samples[-3:]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for (_, _, why, _) in rows for n, m in self.masks if why & m})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(r[1] for r in rows), "reasons": reasons,
                "power_w_median": round(statistics.median(r[3] for r in rows), 1),
                "samples": len(rows), "source": "nvml, 2 ms"}


def clock_sampler(gpu_id):
    """NVML sampler, else the nvidia-smi one."""
    try:
        return NvmlClockSampler(gpu_id)
    except Exception:
        return ClockSampler(gpu_id)


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a window
    (the fallback when NVML is not importable)."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()

    def _reader(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 - 0.15 <= t <= t1 + 0.15] or \
               [s for (_, s) in self.samples[-3:]]
        mhz, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            c = [x.strip() for x in r.split(",")]
            if len(c) < 9:
                continue
            try:
                mhz.append(float(c[1]))
                mx.append(float(c[2]))
            except ValueError:
                continue
            for n, v in zip(names, c[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------- workload building
def build_host(workload, rank, use_oracle_quantizer=False):
    cfg, nblocks, M, projs = WORKLOADS[workload]
    if use_oracle_quantizer:
        import oracle
        q4, q8 = oracle.quant_q4_g32, oracle.quant_q8_row
    else:
        import int8_dequant_gemm_b200 as rtq
        q4, q8 = rtq.quantize_q4_g32, rtq.quantize_q8_row
    blocks = []
    for b in range(nblocks):
        blk = {}
        for name in projs:
            fmt = proj_dims(name)[0]
            W = wl.projection_weights(cfg, b, name)
            blk[name] = q4(W) if fmt == "q4" else q8(W)
            # replicas: same weights, rank-specific activations
            spec = wl.BLOCK_PROJECTIONS[name]
            blk["x_" + name] = wl.activations(M, spec["K"],
                                              wl.seed_for(cfg, b, spec["x"]) + 100_000 * rank)
        blocks.append(blk)
    return cfg, nblocks, M, projs, blocks


def reduce_max(x, world, device):
    """Largest value of x over all ranks (x itself at world size 1): every
    rank's timed region is the job's when the ranks run in lockstep."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, flops_per_rank_step, ms_per_step):
    """Whole-job TFLOP/s: every rank processes its own batch each step."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def step_flops(M, nblocks, projs):
    return nblocks * sum(proj_flops(p, M) for p in projs)


def step_weight_bytes(nblocks, projs):
    return nblocks * sum(weight_bytes(p) for p in projs)


# ---------------------------------------------------------- CPU baseline
def host_threads():
    """Host cores this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_oracle_sample(blocks, M, projs, rows_per_proj, seed, threads=1):
    """Runs the oracle on `rows_per_proj` seeded rows of every projection,
    the rows split over `threads` host threads (the oracle's C call releases
    the interpreter lock, so the threads run on separate cores); returns
    (seconds, flops)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    rows = wl.sample_rows(M, rows_per_proj, seed)
    parts = [p for p in np.array_split(rows, max(1, min(threads, len(rows)))) if len(p)]
    flops = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(parts)) as pool:
        for blk in blocks:
            for name in projs:
                fmt, N, K = proj_dims(name)
                g = oracle.gemm_q4 if fmt == "q4" else oracle.gemm_q8
                list(pool.map(lambda r: g(blk["x_" + name], *blk[name], rows=r), parts))
                flops += 2 * len(rows) * N * K
    return time.perf_counter() - t0, flops


# ------------------------------------------------------------- reference
def run_reference(args, rank, world):
    """The CPU oracle, timed on this host's cores, on the same workload."""
    if rank != 0:
        return
    if WORKLOADS[args.workload][1] == 0:
        print(json.dumps({"impl": "reference", "unavailable":
                          f"the oracle arm times the block workloads; {args.workload} has none"}),
              flush=True)
        return
    cfg, nblocks, M, projs, blocks = build_host(args.workload, 0, use_oracle_quantizer=True)
    threads = host_threads()
    rows = max(args.ref_rows, 2 * threads)
    for i in range(args.warmup):
        cpu_oracle_sample(blocks, M, projs, rows, seed=i, threads=threads)
    secs, flops = 0.0, 0
    for i in range(args.steps):
        s, f = cpu_oracle_sample(blocks, M, projs, rows, seed=1000 + i, threads=threads)
        secs += s
        flops += f
    value = flops / secs / 1e12
    sample = (f"{rows} seeded rows of M={M} per projection, {nblocks} block(s) x "
              f"{len(projs)} projections per step, rows split over {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "blocks": nblocks, "M": M,
                   "projections": list(projs), "rows_sampled_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ timing helpers
def gpu_uuid(dev, local_rank):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return local_rank


def graph_time_us(stream, fn, reps, steps, warmup):
    """Device time of one call of fn(): `reps` back-to-back calls captured in
    one CUDA graph, `steps` replays between CUDA events on `stream` (after
    `warmup` replays); the first call runs outside the capture."""
    import torch
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            fn()
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 1)):
            g.replay()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (steps * reps)


def roofline(flops, nbytes, seconds, peaks, sustained=False):
    """Roofline object of work that moves `nbytes` of algorithmic HBM traffic
    and does `flops` in `seconds`.  The bound is the binding side of
    min(tensor peak, flops/byte x HBM peak): "hbm" reports GB/s against the
    measured copy bandwidth, "tensor" TFLOP/s against the measured dense peak
    (the fp16 MMA runs at the bf16 rate, nominal ratio 1; the burst figure for
    work timed in short windows, the sustained one for seconds-long loops)."""
    tc = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    intensity = flops / nbytes
    attainable = min(tc, intensity * hbm / 1e3)             # TFLOP/s
    if intensity * hbm / 1e3 <= tc:
        r = {"bound": "hbm", "achieved": nbytes / seconds / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        r = {"bound": "tensor", "achieved": flops / seconds / 1e12, "peak": tc, "unit": "TFLOP/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r.update({"algorithmic_flops": flops, "algorithmic_bytes": nbytes,
              "flop_per_byte": intensity, "attainable_tflops": attainable,
              "tflops": flops / seconds / 1e12,
              "tensor_peak": "sustained" if sustained else "burst",
              "peak_source": peaks["source"]})
    return r


# --------------------------------------------------------- small-M stream
def measure_small_m(args, rank, world, local_rank, dev, stream, blocks=None):
    """Small-M projections measured as an aggregate weight stream.

    One M = 80 projection moves well under a megabyte of weights, less than a
    launch's latency worth, so the small-M rate is measured over many: the 12
    blocks' quantized weights are copied into distinct device buffers until
    the copies total about 4x L2, and one step runs every copy's block
    projection set (qkvg, wo, w13, w2) at M = 80.  The projections go through
    rt_qgemm_batch, `copies_per_call` block copies (4 entries each) per call:
    within a call every entry has its own Y, and the calls reuse one set of
    Y buffers and one X buffer per projection (L2-resident, as the
    activations of a real forward pass are), so the weights are the only
    stream from HBM.  The step is captured once as a CUDA graph and replayed.
    The same copies are also run one rt_qblock_project call per copy (the
    block driver's grouped launch) for comparison.  Returns the measurement
    (value = quantized weight bytes per step / time, GB/s)."""
    import torch
    import torch.distributed as dist

    import int8_dequant_gemm_b200 as rtq

    L = rtq.lib()
    sptr = ctypes.c_void_p(stream.cuda_stream)
    M, projs = 80, ("qkvg", "wo", "w13", "w2")
    cfg = 4
    per_call = args.copies_per_call
    if blocks is None:
        _, _, _, _, blocks = build_host("blocks12_m4096", rank)   # the 12 blocks' weights
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_block = sum(weight_bytes(p) for p in projs)
    copies = max(len(blocks), int(math.ceil(4 * l2 / per_block)))
    copies = (copies + per_call - 1) // per_call * per_call

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    xs = {p: d(wl.activations(M, proj_dims(p)[2], wl.seed_for(cfg, 0, wl.BLOCK_PROJECTIONS[p]["x"])
                                  + 100_000 * rank)) for p in projs}
    ys = [{p: torch.empty((M, proj_dims(p)[1]), dtype=torch.float32, device=dev) for p in projs}
          for _ in range(per_call)]
    dev_blocks = []
    for c in range(copies):
        blk = blocks[c % len(blocks)]
        dev_blocks.append({p: tuple(d(a) for a in blk[p]) for p in projs})   # distinct copies
    # one rt_qproj array per call: per_call copies x 4 projections
    arrays = []
    for c0 in range(0, copies, per_call):
        arr = (rtq._QProjC * (4 * per_call))()
        for j in range(per_call):
            db = dev_blocks[c0 + j]
            for k, p in enumerate(projs):
                N, K = proj_dims(p)[1:]
                arr[4 * j + k] = rtq._QProjC(4 if proj_dims(p)[0] == "q4" else 8, 0,
                                             xs[p].data_ptr(), db[p][0].data_ptr(),
                                             db[p][1].data_ptr(), None, ys[j][p].data_ptr(), N, K)
        arrays.append(arr)
    route = rtq.KERNELS.get(L.rt_qgemm_batch_plan(arrays[0], 4 * per_call, M, 0), "per call")
    structs = [rtq._QBlockC(*(t.data_ptr() for p in projs for t in db[p]), wl.D_MODEL, wl.D_FF)
               for db in dev_blocks]
    xptr = [xs[p].data_ptr() for p in projs]
    yptr = [ys[0][p].data_ptr() for p in projs]

    def step_batch():
        for arr in arrays:
            st = L.rt_qgemm_batch(arr, 4 * per_call, M, 0, sptr)
            if st:
                raise rtq.RtqError(st, "rt_qgemm_batch")

    def step_blocks():
        for c in structs:
            st = L.rt_qblock_project(ctypes.byref(c), M, *xptr, *yptr, 0, sptr)
            if st:
                raise rtq.RtqError(st, "rt_qblock_project")

    def timed(step, sample_clocks):
        with torch.cuda.stream(stream):
            for _ in range(2):
                step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 1)):
                graph.replay()
        stream.synchronize()
        if rtq.device_status(stream) != 0:
            raise RuntimeError("device status word reports a fault during the small-M warm-up")
        sampler = clock_sampler(gpu_uuid(dev, local_rank)) if sample_clocks else None
        if sampler:
            sampler.start()
            time.sleep(0.3)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(dev)
        t0 = time.time()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        t1 = time.time()
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        clocks = None
        if sampler:
            sampler.stop()
            clocks = sampler.summary(t0, t1)
        ms = reduce_max(e0.elapsed_time(e1), world, dev) / args.steps
        if rtq.device_status(stream) != 0:
            raise RuntimeError("device status word reports a fault in the small-M stream")
        del graph
        return ms, clocks

    ms, clocks = timed(step_batch, True)
    ms_blocks, _ = timed(step_blocks, False)
    wbytes = copies * per_block
    flops = copies * sum(proj_flops(p, M) for p in projs)
    abytes = copies * sum(proj_bytes(p, M) for p in projs)
    peaks = load_peaks()
    gbs = world * wbytes / (ms * 1e-3) / 1e9
    n_calls = len(arrays)
    launches_per_call = (1 + int(math.ceil(4 * per_call / 256))) if route == "tc_list" else None
    return {
        "metric": "quantized weight GB/s at M = 80 (aggregate stream)", "value": gbs,
        "unit": "GB/s", "ms_per_step": ms, "steps": args.steps,
        "frac_of_hbm": gbs / world / peaks["hbm_gbs"], "hbm_peak_gbs": peaks["hbm_gbs"],
        "tflops": world * flops / (ms * 1e-3) / 1e12,
        "config": {"workload": "rot_m80", "M": M, "projections": list(projs),
                   "weight_copies": copies, "copies_per_call": per_call,
                   "calls_per_step": n_calls, "weight_bytes_per_step": wbytes,
                   "route": route,
                   "l2": f"weights rotate over {wbytes / 1e6:.0f} MB ({wbytes / l2:.1f}x L2); "
                         f"X and Y reused by every call (L2-resident)",
                   "replay": "CUDA graph of the step's rt_qgemm_batch calls"},
        "gpu_launches": args.steps * n_calls * launches_per_call if launches_per_call else None,
        "grouped_block_launch_gbs": world * wbytes / (ms_blocks * 1e-3) / 1e9,
        "roofline_weights_only": {"bound": "hbm", "achieved": gbs / world,
                                  "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / world / peaks["hbm_gbs"],
                                  "peak_source": peaks["source"]},
        "roofline": roofline(flops, abytes, ms * 1e-3, peaks),
        "clocks": clocks,
    }


def run_small_m(args, rank, world, local_rank):
    """The rot_m80 workload on its own, printed as one JSON line."""
    import torch
    import int8_dequant_gemm_b200 as rtq
    rtq.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    r = measure_small_m(args, rank, world, local_rank, dev, stream)
    if rank == 0:
        line = {
            "metric": METRIC, "value": r["value"], "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "accumulate": "f32", "data": "synthetic",
            "config": dict(r["config"],
                           parallelism=f"replicas{world}" if world > 1 else "single"),
            "tflops": r["tflops"], "clocks": r["clocks"], "gpu_launches": r["gpu_launches"],
            "roofline": dict(r["roofline_weights_only"], traffic=None),
            "roofline_all_bytes": r["roofline"], "e2e": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ large M gate
def measure_large_m(args, rank, world, local_rank, dev, stream):
    """The large-M gate: q4 512->2048 (the ffn.w1 shape) at M = 65536 (B = 64,
    S = 1024) with a seeded 1 % of groups holding a x20 outlier, RT_PATH_AUTO,
    five calls per CUDA graph.  X (128 MiB) and Y (512 MiB) exceed L2."""
    import torch
    import torch.distributed as dist

    import int8_dequant_gemm_b200 as rtq

    L = rtq.lib()
    sptr = ctypes.c_void_p(stream.cuda_stream)
    M, N, K = 65536, 2048, 512
    seed = wl.seed_for(5, 0, 1)
    W = wl.with_outliers(wl.weights(N, K, seed), seed + 1)
    Wq, S = rtq.quantize_q4_g32(W)
    Wd = torch.from_numpy(Wq).to(dev)
    Sd = torch.from_numpy(S).to(dev)
    X = torch.from_numpy(wl.activations(M, K, seed + 2 + M + 100_000 * rank)).to(dev)
    Y = torch.empty((M, N), dtype=torch.float32, device=dev)
    a = (X.data_ptr(), Wd.data_ptr(), Sd.data_ptr(), Y.data_ptr(), M, N, K, 0, sptr)

    def call():
        st = L.rt_qgemm_q4(*a)
        if st:
            raise rtq.RtqError(st, "rt_qgemm_q4")

    sampler = clock_sampler(gpu_uuid(dev, local_rank))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
    t0 = time.time()
    us = graph_time_us(stream, call, reps=5, steps=max(2, args.steps // 2), warmup=args.warmup)
    t1 = time.time()
    sampler.stop()
    us = reduce_max(us, world, dev)
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a fault in the large-M gate")
    flops = 2 * M * N * K
    nbytes = Wq.nbytes + S.nbytes + 4 * M * K + 4 * M * N
    peaks = load_peaks()
    r = roofline(flops, nbytes, us * 1e-6, peaks)
    del X, Y
    torch.cuda.empty_cache()
    return {
        "metric": "TFLOP/s of q4 512->2048 at M = 65536", "value": world * flops / (us * 1e-6) / 1e12,
        "unit": "TFLOP/s", "us_per_call": us,
        "frac_of_dense_peak": flops / (us * 1e-6) / 1e12 / peaks["bf16_tflops"],
        "dense_peak_tflops": peaks["bf16_tflops"], "kernel": rtq.plan(4, M, N, K),
        "launches_per_call": 1 if rtq.plan(4, M, N, K) == "tc_x_resident_pair" else 2,
        "config": {"shape": "q4 512->2048", "M": M, "path": "auto", "calls_per_graph": 5,
                   "outliers": "1% of groups x20", "l2": "X 128 MiB + Y 512 MiB > L2"},
        "roofline": r, "clocks": sampler.summary(t0, t1),
    }


# --------------------------------------------------------------- M sweep
SWEEP_SHAPES = (("q4", 2048, 512), ("q8", 512, 2048))    # ffn.w1 and ffn.w2 shapes
SWEEP_M = (1, 2, 4, 8, 16, 32, 80, 512, 4096, 65536)
SWEEP_SIMT_MAX_M = 4096      # the fp32 SIMT path is timed up to here


def run_sweep(args, rank, world, local_rank):
    """M sweep of the q4 512->2048 and q8 2048->512 projections (weights with a
    seeded 1 % of 32-groups holding a x20 outlier) on the SIMT path, the
    tensor-core path and RT_PATH_AUTO.  Every point streams from HBM: the
    weights, activations and outputs are held in as many copies as make at
    least 2x L2, and successive calls use successive copies (a CUDA graph of
    max(copies, 20) calls).  `crossover` gives, per shape, the smallest M at
    which the tensor-core path beats the SIMT path; value = TFLOP/s of the q4
    shape at M = 65536 (AUTO), the large-M gate."""
    import torch

    import int8_dequant_gemm_b200 as rtq

    rtq.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)
    L = rtq.lib()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peaks = load_peaks()
    points = []
    for fmt, N, K in SWEEP_SHAPES:
        seed = wl.seed_for(5, 0, 1 if fmt == "q4" else 3)
        W = wl.with_outliers(wl.weights(N, K, seed), seed + 1)
        Wq, S = rtq.quantize_q4_g32(W) if fmt == "q4" else rtq.quantize_q8_row(W)
        fn = L.rt_qgemm_q4 if fmt == "q4" else L.rt_qgemm_q8
        fcode = 4 if fmt == "q4" else 8
        wb = Wq.nbytes + S.nbytes
        for M in SWEEP_M:
            per_copy = wb + 4 * M * K + 4 * M * N
            copies = max(1, min(1000, int(math.ceil(2 * l2 / per_copy))))
            X0 = wl.activations(M, K, seed + 2 + M)
            bufs = []
            for _ in range(copies):
                bufs.append((torch.from_numpy(X0).to(dev), torch.from_numpy(Wq).to(dev),
                             torch.from_numpy(S).to(dev),
                             torch.empty((M, N), dtype=torch.float32, device=dev)))
            reps = max(copies, 20)
            for path, pcode in (("simt", 1), ("tc", 2), ("auto", 0)):
                if path == "simt" and M > SWEEP_SIMT_MAX_M:
                    continue
                args_list = [(x.data_ptr(), w.data_ptr(), sc.data_ptr(), y.data_ptr(), M, N, K,
                              pcode, sptr) for x, w, sc, y in bufs]
                state = {"i": 0}

                def call():
                    st = fn(*args_list[state["i"] % copies])
                    state["i"] += 1
                    if st:
                        raise rtq.RtqError(st, "rt_qgemm")

                us = graph_time_us(stream, call, reps=reps, steps=args.steps, warmup=args.warmup)
                points.append({
                    "shape": f"{fmt} {K}->{N}", "M": M, "path": path,
                    "kernel": rtq.plan(fcode, M, N, K, path), "us_per_call": us,
                    "tflops": 2.0 * M * N * K / (us * 1e-6) / 1e12,
                    "weight_gbs": wb / (us * 1e-6) / 1e9,
                    "roofline": roofline(2.0 * M * N * K, per_copy, us * 1e-6, peaks),
                    "copies": copies})
            del bufs
            torch.cuda.empty_cache()
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a fault")
    crossover = {}
    for fmt, N, K in SWEEP_SHAPES:
        name = f"{fmt} {K}->{N}"
        won = [M for M in SWEEP_M
               if any(p["shape"] == name and p["M"] == M and p["path"] == "simt" for p in points)
               and next(p for p in points if p["shape"] == name and p["M"] == M
                        and p["path"] == "tc")["us_per_call"]
               < next(p for p in points if p["shape"] == name and p["M"] == M
                      and p["path"] == "simt")["us_per_call"]]
        crossover[name] = {"tc_faster_from_M": min(won) if won else None,
                           "auto_simt_max_M": max(M for M in range(1, 129)
                                                  if rtq.auto_path(fmt == "q4" and 4 or 8, M, N, K) == 1)}
    head = next(p for p in points if p["shape"].startswith("q4") and p["M"] == SWEEP_M[-1]
                and p["path"] == "auto")
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["tflops"], "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["us_per_call"] * 1e-3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "accumulate": "f32", "data": "synthetic",
            "config": {"workload": "m_sweep", "shapes": [f"{f} {k}->{n}" for f, n, k in SWEEP_SHAPES],
                       "M": list(SWEEP_M), "paths": ["simt", "tc", "auto"],
                       "simt_max_M": SWEEP_SIMT_MAX_M,
                       "l2": "weights, X and Y in >= 2x L2 of rotating copies"},
            "roofline": dict(head["roofline"], traffic=None),
            "crossover": crossover, "sweep": points, "e2e": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import int8_dequant_gemm_b200 as rtq
    from int8_dequant_gemm_b200 import build as rtq_build

    if not os.path.exists(rtq.LIB_PATH):
        rtq_build.build()
    rtq.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)

    cfg, nblocks, M, projs, blocks = build_host(args.workload, rank)
    L = rtq.lib()

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # device buffers and raw ABI argument lists (marshalled once)
    dblocks, calls = [], []
    for blk in blocks:
        db = {}
        for name in projs:
            fmt, N, K = proj_dims(name)
            Wq, S = (d(a) for a in blk[name])
            X = d(blk["x_" + name])
            Y = torch.empty((M, N), dtype=torch.float32, device=dev)
            db[name] = (Wq, S, X, Y)
            fn = L.rt_qgemm_q4 if fmt == "q4" else L.rt_qgemm_q8
            calls.append((name, fn, (X.data_ptr(), Wq.data_ptr(), S.data_ptr(), Y.data_ptr(),
                                     M, N, K, 0, sptr)))
        dblocks.append(db)
    full_block = tuple(projs) == ("qkvg", "wo", "w13", "w2")
    # the mixed recipe goes through rt_qblock_project, a one-format workload
    # through rt_qblock_project_fmt
    per_fmt = bool(FORMAT_OVERRIDE)
    block_args = []
    if full_block:
        for db in dblocks:
            if per_fmt:
                ws = [rtq._QWeightC(4 if proj_dims(n)[0] == "q4" else 8, 0, db[n][0].data_ptr(),
                                    db[n][1].data_ptr(), None) for n in projs]
                c = rtq._QBlockFmtC(*ws, wl.D_MODEL, wl.D_FF)
            else:
                c = rtq._QBlockC(*(t.data_ptr() for t in (db["qkvg"][0], db["qkvg"][1],
                                                          db["wo"][0], db["wo"][1], db["w13"][0],
                                                          db["w13"][1], db["w2"][0], db["w2"][1])),
                                 wl.D_MODEL, wl.D_FF)
            block_args.append((c, [db[n][2].data_ptr() for n in projs] +
                               [db[n][3].data_ptr() for n in projs]))
    block_fn = L.rt_qblock_project_fmt if per_fmt else L.rt_qblock_project

    def run_block(i):
        c, ptrs = block_args[i]
        st = block_fn(ctypes.byref(c), M, *ptrs, 0, sptr)
        if st:
            raise rtq.RtqError(st, "rt_qblock_project")

    def step():
        if full_block:
            for i in range(len(block_args)):
                run_block(i)
        else:
            for _, fn, a in calls:
                st = fn(*a)
                if st:
                    raise rtq.RtqError(st, "rt_qgemm")

    # the TMA-fed kernels add an activation pre-pass launch; the block driver
    # runs a small-M block as one grouped launch, and above 128 rows the
    # projections that take the one-CTA activation-resident kernel (if two or
    # more do) as one pre-pass launch and one launch of that kernel
    def plan_of(name):
        fmt, N, K = proj_dims(name)
        return rtq.plan(4 if fmt == "q4" else 8, M, N, K)

    def call_launches_of(name):
        return 2 if plan_of(name) in ("tc_x_resident", "tc_w_streamed") else 1

    if full_block and per_fmt:
        fused_block = L.rt_qblock_fused_fmt(ctypes.byref(block_args[0][0]), M, 0) == 1
    else:
        fused_block = full_block and rtq.block_fused(M, wl.D_MODEL, wl.D_FF) == 1
    # the block driver's route (rt_qblock_route): which launches a block takes
    route_names = []
    if full_block:
        c0 = block_args[0][0]
        bits = (L.rt_qblock_route_fmt if per_fmt else L.rt_qblock_route)(ctypes.byref(c0), M, 0)
        route_names = [n for b, n in ((rtq.ROUTE_GROUPED_SMALL_M, "grouped_small_m"),
                                      (rtq.ROUTE_X_RESIDENT_GROUP, "x_resident_group"),
                                      (rtq.ROUTE_SIDE_PREPASS, "side_stream_prepass"))
                       if bits >= 0 and bits & b] or ["one_call_per_projection"]
    grouped = []
    if full_block and not fused_block:
        grouped = [n for n in projs if plan_of(n) == "tc_x_resident"]
        if len(grouped) < 2:
            grouped = []
    if fused_block:
        launches_per_step = nblocks
    elif full_block:
        launches_per_step = nblocks * ((2 if grouped else 0) +
                                       sum(call_launches_of(n) for n in projs if n not in grouped))
    else:
        launches_per_step = sum(call_launches_of(name) for name, _, _ in calls)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    # ---- warm-up
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 1)):
            step()
    stream.synchronize()
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a fault during warm-up")

    # ---- the step captured once as a CUDA graph, so that the host's cost of
    # issuing the step's launches stays out of the timed region; if the capture is
    # refused, the step is issued call by call instead (named in config.issue)
    graph, issue = None, "eager"
    if not args.eager:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step()
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
            if rtq.device_status(stream) != 0:
                raise RuntimeError("fault in the captured step")
            graph, issue = g, "cuda_graph"
        except Exception as exc:   # fall back to eager issue, recorded in the line
            torch.cuda.synchronize(dev)
            graph, issue = None, f"eager (graph capture failed: {type(exc).__name__})"

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            step()

    # ---- timed region: K steps through the block driver
    sampler = clock_sampler(gpu_uuid(dev, local_rank))
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            run_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier()
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    ms_per_step = ms_total / args.steps
    del graph

    # ---- per-call device time, each call of block 0 in its own CUDA graph of
    # 20 back-to-back calls (a block run as one grouped launch is timed as
    # that launch); the sum over the step is checked against ms_per_step
    reps = 20
    group_key = "+".join(grouped)
    if fused_block:
        kern_us = {"block": graph_time_us(stream, lambda: run_block(0), reps, args.steps,
                                          args.warmup)}
    else:
        kern_us = {}
        if grouped:
            # block 0's grouped projections as the block driver runs them: an
            # rt_qgemm_batch list above 128 rows takes the same grouped launch
            garr = (rtq._QProjC * len(grouped))()
            for i, n in enumerate(grouped):
                fmt, N, K = proj_dims(n)
                Wq, S, X, Y = dblocks[0][n]
                garr[i] = rtq._QProjC(4 if fmt == "q4" else 8, 0, X.data_ptr(), Wq.data_ptr(),
                                      S.data_ptr(), None, Y.data_ptr(), N, K)

            def group_call():
                st = L.rt_qgemm_batch(garr, len(grouped), M, 0, sptr)
                if st:
                    raise rtq.RtqError(st, "rt_qgemm_batch")
            kern_us[group_key] = graph_time_us(stream, group_call, reps, args.steps, args.warmup)
        for name, fn, a in calls[:len(projs)]:
            if name in grouped:
                continue

            def one(fn=fn, a=a):
                st = fn(*a)
                if st:
                    raise rtq.RtqError(st, "rt_qgemm")
            kern_us[name] = graph_time_us(stream, one, reps, args.steps, args.warmup)
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a fault")

    flops = step_flops(M, nblocks, projs)
    value = job_value(world, flops, ms_per_step)
    wbytes = step_weight_bytes(nblocks, projs)

    # ---- roofline of the dominant call
    peaks = load_peaks()
    if fused_block:
        share = {"block": kern_us["block"] * nblocks}
        dom, path = "block", "tc"
        b_alg = sum(proj_bytes(p, M) for p in projs)
        f_alg = sum(proj_flops(p, M) for p in projs)
        kernel_key = f"block_grouped_tc_M{M}"
        call_launches = 1
    else:
        share = {n: kern_us[n] * nblocks for n in kern_us}
        dom = max(share, key=share.get)
        if dom == group_key:
            b_alg = sum(proj_bytes(p, M) for p in grouped)
            f_alg = sum(proj_flops(p, M) for p in grouped)
            kernel_key = f"group_{group_key}_M{M}"
            call_launches = 2
        else:
            fmt, N, K = proj_dims(dom)
            fcode = 4 if fmt == "q4" else 8
            path = "tc" if rtq.auto_path(fcode, M, N, K) == 2 else "simt"
            b_alg, f_alg = proj_bytes(dom, M), proj_flops(dom, M)
            kernel_key = f"{dom}_{fmt}_{path}_M{M}"
            call_launches = call_launches_of(dom)
    if dom == "block":
        dom_plan = "tc_w_stationary (grouped)"
    elif dom == group_key:
        dom_plan = "tc_x_resident (one launch for " + ", ".join(grouped) + ")"
    else:
        dom_plan = plan_of(dom)
    roof = roofline(f_alg, b_alg, kern_us[dom] * 1e-6, peaks)
    roof.update({"traffic": recorded_traffic(kernel_key), "kernel": kernel_key,
                 "kernel_plan": dom_plan,
                 "launches_per_call": call_launches, "avg_call_us": kern_us[dom],
                 "timed_as": "one call, 20 per CUDA graph, mean over replays",
                 "share_of_step": share[dom] / sum(share.values())})
    calls_sum_ms = sum(share.values()) * 1e-3

    # ---- end to end: pinned host inputs in, results out, inside the timed region
    e2e = None
    if not args.no_e2e:
        hx, hy = [], []
        for db in dblocks:
            for name in projs:
                Wq, S, X, Y = db[name]
                hx.append((torch.empty(X.shape, dtype=X.dtype, pin_memory=True).copy_(X.cpu()), X))
                hy.append((torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True), Y))
        h2d = sum(h.numel() * 4 for h, _ in hx)
        d2h = sum(h.numel() * 4 for h, _ in hy)
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)
        nproj = len(projs)

        def e2e_step():
            """One step end to end.  With whole blocks, block by block on three
            streams: block i's inputs are copied in on s_in while earlier blocks
            compute, block i runs on the ABI's stream once they have landed, and
            its outputs are copied out on s_out while later blocks compute (PCIe
            carries both directions at once); the streams join at the end of the
            step.  Otherwise all inputs in, the step, all outputs out."""
            if not full_block:
                with torch.cuda.stream(stream):
                    for h, dv in hx:
                        dv.copy_(h, non_blocking=True)
                    step()
                    for h, dv in hy:
                        h.copy_(dv, non_blocking=True)
                return
            start = torch.cuda.Event()
            start.record(stream)
            s_in.wait_event(start)
            s_out.wait_event(start)
            for i in range(len(block_args)):
                landed = torch.cuda.Event()
                with torch.cuda.stream(s_in):
                    for h, dv in hx[i * nproj:(i + 1) * nproj]:
                        dv.copy_(h, non_blocking=True)
                    landed.record(s_in)
                stream.wait_event(landed)
                with torch.cuda.stream(stream):
                    run_block(i)
                done = torch.cuda.Event()
                done.record(stream)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    for h, dv in hy[i * nproj:(i + 1) * nproj]:
                        h.copy_(dv, non_blocking=True)
            out_done = torch.cuda.Event()
            out_done.record(s_out)
            stream.wait_event(out_done)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1)) / n_e2e
        e2e = {"value": job_value(world, flops, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "steps": n_e2e,
               "copies": ("per block on two copy streams beside the compute stream"
                          if full_block else "all inputs, the step, all outputs, one stream")}
        del hx, hy

    # ---- the two gates of the metric, measured in the same run on the
    # default workload: small M (aggregate weight stream) and M = 65536
    small_m = large_m = None
    if args.workload == "blocks12_m4096" and not args.no_gates:
        del dblocks, calls, block_args
        torch.cuda.empty_cache()
        small_m = measure_small_m(args, rank, world, local_rank, dev, stream, blocks=blocks)
        torch.cuda.empty_cache()
        large_m = measure_large_m(args, rank, world, local_rank, dev, stream)

    # ---- CPU oracle baseline on a bounded sample (rank 0, single GPU only)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        threads = host_threads()
        rows = max(args.cpu_rows, 16 * threads)
        secs, cflops = cpu_oracle_sample(blocks, M, projs, rows, seed=7, threads=threads)
        cpu = {"value": cflops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} seeded rows of M={M} for each of the "
                         f"{nblocks * len(projs)} projections ({cflops / 1e9:.2f} GFLOP, "
                         f"{secs:.1f} s, double-precision oracle, rows split over {threads} "
                         f"host threads)"}

    if rank == 0:
        bytes_act = sum(4 * M * (proj_dims(p)[1] + proj_dims(p)[2]) for p in projs) * nblocks
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "accumulate": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "blocks": nblocks, "M": M,
                       "projections": list(projs), "d_model": wl.D_MODEL, "d_ff": wl.D_FF,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": f"inputs > L2 ({(bytes_act + wbytes) / 1e9:.2f} GB streamed per "
                             f"step), no flush",
                       "issue": issue, "block_route": route_names},
            "weight_gbs": world * wbytes / (ms_per_step * 1e-3) / 1e9,
            "call_us": kern_us, "calls_sum_ms_per_step": calls_sum_ms,
            "clocks": clocks, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "roofline": roof, "cpu_baseline": cpu,
            "small_m": small_m, "large_m": large_m,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("rtq", "reference"), default="rtq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="blocks12_m4096")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-rows", type=int, default=128,
                    help="rows per projection in the CPU-oracle sample")
    ap.add_argument("--ref-rows", type=int, default=8,
                    help="rows per projection per step in the reference arm")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="issue the timed steps call by call instead of replaying a CUDA graph")
    ap.add_argument("--copies-per-call", type=int, default=16,
                    help="block copies per rt_qgemm_batch call in the small-M stream")
    ap.add_argument("--no-gates", action="store_true",
                    help="skip the small-M and M = 65536 measurements of the default workload")
    args = ap.parse_args()
    if args.cpu_rows < 2 or args.ref_rows < 2:
        ap.error("--cpu-rows and --ref-rows take at least 2 (rows 0 and M-1 are always sampled)")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in ALL_FORMAT:
        FORMAT_OVERRIDE.update({p: ALL_FORMAT[args.workload] for p in wl.BLOCK_PROJECTIONS})
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "rot_m80":
            run_small_m(args, rank, world, local_rank)
        elif args.workload == "m_sweep":
            run_sweep(args, rank, world, local_rank)
        else:
            run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
