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
             memory and its outputs copied back inside the timed region;
  roofline   the dominant kernel (the projection with the largest share of the
             step), its algorithmic bytes or flops per launch over its
             CUDA-event duration, against MEASURED_PEAKS.json;
  cpu_baseline  the CPU oracle on a bounded row sample of the same workload.

`--impl reference` times the CPU oracle itself (rank 0 only) on the same
workload, metric and unit, one bounded row sample per step.

Other workloads (`--workload`), each printing one line of the same form:
  block_m80, block_m2048
               one block's projection set at M = 80 (one grouped launch; the
               roofline object then describes that launch) and at M = 2048.
  rot_m80      small M as an aggregate weight stream: the 12 blocks' weights in
               rotating device copies totalling ~4x L2, every copy's projection
               set at M = 80, replayed from a CUDA graph; value in GB/s of
               quantized weights.
  m_sweep      M in {1, 16, 80, 512, 4096, 65536} for the q4 512->2048 and q8
               2048->512 shapes under the automatic dispatch; value = TFLOP/s
               of the q4 shape at M = 65536, every point under `sweep`.
  w13_m4096, w2_m4096, qkvg_m4096, w13_m16384, w2_m16384
               single projections, sized for profiler captures.

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
}


def proj_dims(name):
    spec = wl.BLOCK_PROJECTIONS[name]
    return spec["fmt"], spec["N"], spec["K"]


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


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a window."""
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
            fmt = wl.BLOCK_PROJECTIONS[name]["fmt"]
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
def cpu_oracle_sample(blocks, M, projs, rows_per_proj, seed):
    """Runs the oracle on `rows_per_proj` seeded rows of every projection;
    returns (seconds, flops)."""
    import oracle
    rows = wl.sample_rows(M, rows_per_proj, seed)
    flops = 0
    t0 = time.perf_counter()
    for blk in blocks:
        for name in projs:
            fmt, N, K = proj_dims(name)
            g = oracle.gemm_q4 if fmt == "q4" else oracle.gemm_q8
            g(blk["x_" + name], *blk[name], rows=rows)
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
    rows = args.ref_rows
    for i in range(args.warmup):
        cpu_oracle_sample(blocks, M, projs, rows, seed=i)
    secs, flops = 0.0, 0
    for i in range(args.steps):
        s, f = cpu_oracle_sample(blocks, M, projs, rows, seed=1000 + i)
        secs += s
        flops += f
    value = flops / secs / 1e12
    sample = (f"{rows} seeded rows of M={M} per projection, {nblocks} block(s) x "
              f"{len(projs)} projections per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "blocks": nblocks, "M": M,
                   "projections": list(projs), "rows_sampled_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------- small-M stream
def run_small_m(args, rank, world, local_rank):
    """Small-M projections measured as an aggregate weight stream.

    One M = 80 projection moves well under a megabyte of weights, less than a
    launch's latency worth, so the small-M rate is measured over many: the 12
    blocks' quantized weights are copied into distinct device buffers until the
    copies total about 4x L2, and one step runs every copy's block projection
    set (qkvg, wo, w13, w2) at M = 80 through rt_qblock_project.  X and Y are
    one buffer per projection shared by all copies (L2-resident, as the
    activations of a real forward pass are).  The step is captured once as a
    CUDA graph and replayed.  value = quantized weight bytes per step / time.
    """
    import torch
    import torch.distributed as dist

    import int8_dequant_gemm_b200 as rtq

    rtq.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)
    L = rtq.lib()
    cfg, nblocks, M, projs = WORKLOADS[args.workload]
    _, _, _, _, blocks = build_host("blocks12_m4096", rank)   # the 12 blocks' quantized weights
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_block = sum(weight_bytes(p) for p in projs)
    copies = max(len(blocks), int(math.ceil(4 * l2 / per_block)))

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    xs = {p: d(wl.activations(M, proj_dims(p)[2], wl.seed_for(cfg, 0, wl.BLOCK_PROJECTIONS[p]["x"])
                                  + 100_000 * rank)) for p in projs}
    ys = {p: torch.empty((M, proj_dims(p)[1]), dtype=torch.float32, device=dev) for p in projs}
    dev_blocks, structs = [], []
    for c in range(copies):
        blk = blocks[c % len(blocks)]
        db = {p: tuple(d(a) for a in blk[p]) for p in projs}   # fresh device copy each time
        dev_blocks.append(db)
        structs.append(rtq._QBlockC(*(t.data_ptr() for p in projs for t in db[p]),
                                    wl.D_MODEL, wl.D_FF))
    xptr = [xs[p].data_ptr() for p in projs]
    yptr = [ys[p].data_ptr() for p in projs]

    def step():
        for c in structs:
            st = L.rt_qblock_project(ctypes.byref(c), M, *xptr, *yptr, 0, sptr)
            if st:
                raise rtq.RtqError(st, "rt_qblock_project")

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
        raise RuntimeError("device status word reports a timed-out wait during warm-up")

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    gpu_id = local_rank
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    barrier()
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    ms = reduce_max(e0.elapsed_time(e1), world, dev) / args.steps
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a timed-out wait")
    del graph
    wbytes = copies * per_block
    gbs = world * wbytes / (ms * 1e-3) / 1e9
    flops = copies * sum(proj_flops(p, M) for p in projs)
    peaks = load_peaks()
    kernels = sorted({rtq.plan(4 if proj_dims(p)[0] == "q4" else 8, M, *proj_dims(p)[1:])
                      for p in projs})
    fused = rtq.block_fused(M, wl.D_MODEL, wl.D_FF) == 1
    launches_per_copy = 1 if fused else sum(
        2 if rtq.plan(4 if proj_dims(p)[0] == "q4" else 8, M, *proj_dims(p)[1:])
        in ("tc_x_resident", "tc_w_streamed") else 1 for p in projs)
    if rank == 0:
        line = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accumulate": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload, "M": M, "projections": list(projs),
                       "weight_copies": copies, "weight_bytes_per_step": wbytes,
                       "l2_bytes": l2, "replay": "CUDA graph of all copies' block projection sets",
                       "l2": f"weights rotate over {wbytes / 1e6:.0f} MB ({wbytes / l2:.1f}x L2); "
                             f"X and Y fixed",
                       "parallelism": f"replicas{world}" if world > 1 else "single"},
            "tflops": world * flops / (ms * 1e-3) / 1e12,
            "kernels": kernels, "block_launch": "grouped" if fused else "per projection",
            "clocks": clocks, "gpu_launches": args.steps * copies * launches_per_copy,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_step": wbytes, "peak_source": peaks["source"]},
            "e2e": None, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


# --------------------------------------------------------------- M sweep
SWEEP_SHAPES = (("q4", 2048, 512), ("q8", 512, 2048))    # ffn.w1 and ffn.w2 shapes
SWEEP_M = (1, 16, 80, 512, 4096, 65536)


def run_sweep(args, rank, world, local_rank):
    """M sweep of the q4 512->2048 and q8 2048->512 projections under
    RT_PATH_AUTO (weights with a seeded 1 % of 32-groups holding a x20
    outlier).  Each point is 20 calls captured in a CUDA graph, replayed
    after warm-up; inputs stay in place between calls, so points whose data
    fit in L2 (M <= 4096) run L2-warm.  value = TFLOP/s of the q4 shape at
    M = 65536, the large-M gate; `sweep` lists every point and the kernel the
    dispatcher chose."""
    import torch

    import int8_dequant_gemm_b200 as rtq

    rtq.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)
    L = rtq.lib()
    reps = 20
    points = []
    for fmt, N, K in SWEEP_SHAPES:
        seed = wl.seed_for(5, 0, 1 if fmt == "q4" else 3)
        W = wl.with_outliers(wl.weights(N, K, seed), seed + 1)
        Wq, S = rtq.quantize_q4_g32(W) if fmt == "q4" else rtq.quantize_q8_row(W)
        Wd = torch.from_numpy(Wq).to(dev)
        Sd = torch.from_numpy(S).to(dev)
        fn = L.rt_qgemm_q4 if fmt == "q4" else L.rt_qgemm_q8
        fcode = 4 if fmt == "q4" else 8
        for M in SWEEP_M:
            X = torch.from_numpy(wl.activations(M, K, seed + 2 + M)).to(dev)
            Y = torch.empty((M, N), dtype=torch.float32, device=dev)
            call_args = (X.data_ptr(), Wd.data_ptr(), Sd.data_ptr(), Y.data_ptr(), M, N, K, 0, sptr)

            def calls():
                for _ in range(reps):
                    st = fn(*call_args)
                    if st:
                        raise rtq.RtqError(st, "rt_qgemm")

            with torch.cuda.stream(stream):
                calls()                      # grows the workspace outside the capture
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                calls()
            with torch.cuda.stream(stream):
                for _ in range(max(args.warmup, 1)):
                    g.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            stream.synchronize()
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(args.steps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            del g
            us = e0.elapsed_time(e1) * 1e3 / (args.steps * reps)
            wb = Wq.nbytes + S.nbytes
            points.append({"shape": f"{fmt} {K}->{N}", "M": M, "kernel": rtq.plan(fcode, M, N, K),
                           "us_per_call": us, "tflops": 2.0 * M * N * K / (us * 1e-6) / 1e12,
                           "weight_gbs": wb / (us * 1e-6) / 1e9})
            del X, Y
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a timed-out wait")
    peaks = load_peaks()
    head = next(p for p in points if p["shape"].startswith("q4") and p["M"] == SWEEP_M[-1])
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["tflops"], "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["us_per_call"] * 1e-3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "accumulate": "f32", "data": "synthetic",
            "config": {"workload": "m_sweep", "shapes": [f"{f} {k}->{n}" for f, n, k in SWEEP_SHAPES],
                       "M": list(SWEEP_M), "calls_per_graph": reps, "path": "auto",
                       "l2": "inputs reused between calls: L2-warm for M <= 4096"},
            "roofline": {"bound": "tensor", "achieved": head["tflops"],
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": head["tflops"] / peaks["bf16_tflops_sustained"],
                         "peak_source": peaks["source"]},
            "sweep": points, "e2e": None, "cpu_baseline": None,
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
    block_args = []
    if full_block:
        for db in dblocks:
            c = rtq._QBlockC(*(t.data_ptr() for t in (db["qkvg"][0], db["qkvg"][1], db["wo"][0],
                                                      db["wo"][1], db["w13"][0], db["w13"][1],
                                                      db["w2"][0], db["w2"][1])),
                             wl.D_MODEL, wl.D_FF)
            block_args.append((c, [db[n][2].data_ptr() for n in projs] +
                               [db[n][3].data_ptr() for n in projs]))

    def step():
        if full_block:
            for c, ptrs in block_args:
                st = L.rt_qblock_project(ctypes.byref(c), M, *ptrs, 0, sptr)
                if st:
                    raise rtq.RtqError(st, "rt_qblock_project")
        else:
            for _, fn, a in calls:
                st = fn(*a)
                if st:
                    raise rtq.RtqError(st, "rt_qgemm")

    # the TMA-fed kernels add an activation pre-pass launch; the block driver
    # runs a small-M block as one grouped launch
    fused_block = full_block and rtq.block_fused(M, wl.D_MODEL, wl.D_FF) == 1
    if fused_block:
        launches_per_step = nblocks
    else:
        launches_per_step = sum(
            2 if rtq.plan(4 if proj_dims(name)[0] == "q4" else 8, M, *proj_dims(name)[1:])
            in ("tc_x_resident", "tc_w_streamed") else 1
            for name, _, _ in calls)

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
        raise RuntimeError("device status word reports a timed-out wait during warm-up")

    # ---- the step captured once as a CUDA graph, so that the host's cost of
    # issuing 96 launches stays out of the timed region; if the capture is
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
                raise RuntimeError("timed-out wait in the captured step")
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
    gpu_id = local_rank
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
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
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    ms_per_step = ms_total / args.steps

    # ---- per-kernel durations: every launch bracketed by events, K steps.
    # A block run as one grouped launch is timed as that launch.
    evs = {"block": []} if fused_block else {name: [] for name in projs}
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            if fused_block:
                for c, ptrs in block_args:
                    s0 = torch.cuda.Event(enable_timing=True)
                    s1 = torch.cuda.Event(enable_timing=True)
                    s0.record(stream)
                    st = L.rt_qblock_project(ctypes.byref(c), M, *ptrs, 0, sptr)
                    s1.record(stream)
                    if st:
                        raise rtq.RtqError(st, "rt_qblock_project")
                    evs["block"].append((s0, s1))
                continue
            for name, fn, a in calls:
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                fn(*a)
                s1.record(stream)
                evs[name].append((s0, s1))
    torch.cuda.synchronize(dev)
    t_wall2 = time.time()
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall2)
    kern_us = {n: 1e3 * statistics.mean(a.elapsed_time(b) for a, b in v) for n, v in evs.items()}
    if rtq.device_status(stream) != 0:
        raise RuntimeError("device status word reports a timed-out wait")

    flops = step_flops(M, nblocks, projs)
    value = job_value(world, flops, ms_per_step)
    wbytes = step_weight_bytes(nblocks, projs)

    # ---- roofline of the dominant kernel
    peaks = load_peaks()
    if fused_block:
        # one launch per block: its bytes and flops are the four projections'
        share = {"block": kern_us["block"] * nblocks}
        dom, path = "block", "tc"
        b_alg = sum(proj_bytes(p, M) for p in projs)
        f_alg = sum(proj_flops(p, M) for p in projs)
        kernel_key = f"block_grouped_tc_M{M}"
    else:
        share = {n: kern_us[n] * nblocks for n in projs}
        dom = max(share, key=share.get)
        fmt, N, K = proj_dims(dom)
        path = "tc" if rtq.auto_path(4 if fmt == "q4" else 8, M, N, K) == 2 else "simt"
        b_alg, f_alg = proj_bytes(dom, M), proj_flops(dom, M)
        kernel_key = f"{dom}_{fmt}_{path}_M{M}"
    t_s = kern_us[dom] * 1e-6
    t_hbm = b_alg / (peaks["hbm_gbs"] * 1e9)
    t_tc = f_alg / (peaks["bf16_tflops_sustained"] * 1e12)
    traffic = recorded_traffic(kernel_key)
    if t_hbm >= t_tc or path == "simt":
        roof = {"bound": "hbm", "achieved": b_alg / t_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": f_alg / t_s / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
    roof.update({"frac": roof["achieved"] / roof["peak"], "traffic": traffic,
                 "kernel": kernel_key, "algorithmic_bytes": b_alg, "algorithmic_flops": f_alg,
                 "avg_launch_us": kern_us[dom], "peak_source": peaks["source"],
                 "share_of_step": share[dom] / sum(share.values())})

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
        with torch.cuda.stream(stream):
            for h, dv in hx:
                dv.copy_(h, non_blocking=True)
            step()
            for h, dv in hy:
                h.copy_(dv, non_blocking=True)
        torch.cuda.synchronize(dev)
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            f0.record(stream)
            for _ in range(n_e2e):
                for h, dv in hx:
                    dv.copy_(h, non_blocking=True)
                step()
                for h, dv in hy:
                    h.copy_(dv, non_blocking=True)
            f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1)) / n_e2e
        e2e = {"value": job_value(world, flops, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "steps": n_e2e}

    # ---- CPU oracle baseline on a bounded sample (rank 0, single GPU only)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        secs, cflops = cpu_oracle_sample(blocks, M, projs, args.cpu_rows, seed=7)
        cpu = {"value": cflops / secs / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": f"{args.cpu_rows} seeded rows of M={M} for each of the "
                         f"{nblocks * len(projs)} projections ({cflops / 1e9:.2f} GFLOP, "
                         f"{secs:.1f} s, single-threaded double-precision oracle)"}

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
                       "issue": issue},
            "weight_gbs": world * wbytes / (ms_per_step * 1e-3) / 1e9,
            "kernel_us": kern_us,
            "clocks": clocks, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "roofline": roof, "cpu_baseline": cpu,
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
    args = ap.parse_args()
    if args.cpu_rows < 2 or args.ref_rows < 2:
        ap.error("--cpu-rows and --ref-rows take at least 2 (rows 0 and M-1 are always sampled)")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
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
