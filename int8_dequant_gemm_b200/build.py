"""Builds librtq.so (the CUDA library behind include/rtq.h) in-tree for sm_100a.

nvcc compiles the .cu sources with `-gencode arch=compute_100a,code=sm_100a`
(the CUDA runtime is linked statically); g++ compiles the host quantizer with
`-ffp-contract=off` so its double arithmetic is exactly the stated spec.
Objects go to _build/ at the repository root; the library lands next to this
file.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "librtq.so")
HEADER = os.path.join(ROOT, "include", "rtq.h")

CU_SOURCES = ["api.cu", "simt.cu", "tc.cu", "xs.cu", "xp.cu", "ws.cu", "prep.cu", "pl.cu",
              "noalloc.cu"]
CPP_SOURCES = ["quantize.cpp", "st_loader.cpp"]
NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                     "-Xptxas", "-warn-spills", "--expt-relaxed-constexpr"]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-ffp-contract=off", "-fno-fast-math", "-Wall",
             "-Wextra", "-pthread"]


def _deps():
    out = [HEADER]
    for f in os.listdir(CSRC):
        if f.endswith((".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    deps = _deps()
    objs, jobs = [], []
    for src in CU_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + deps):
            cmd = [NVCC] + NVCC_FLAGS + ["-c", s, "-o", o]
            jobs.append((cmd, o))
    for src in CPP_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + deps):
            jobs.append((["g++"] + CXX_FLAGS + ["-c", s, "-o", o], o))
    procs = []
    for cmd, o in jobs:
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT), cmd))
    failed = []
    for p, cmd in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed.append((cmd, text))
        elif verbose and text.strip():
            print(text, flush=True)
    if failed:
        msg = "\n".join(" ".join(c) + "\n" + t for c, t in failed)
        raise RuntimeError("librtq build failed:\n" + msg)
    if force or jobs or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-Xcompiler", "-pthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
