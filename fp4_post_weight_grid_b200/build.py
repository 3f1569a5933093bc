"""Build libfp4q.so in-tree with nvcc for sm_100a.

Flags: -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo and --fmad=false,
given to both the compiler and ptxas (no multiply-add contraction anywhere, so
every binary32 operation is the separately rounded one the results are defined
by).  ptxas resource usage of
every kernel is written to _build/ptxas.log.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp4q.so")
SOURCES = ["api.cu", "absmax.cu", "nvfp4.cu", "mxfp4.cu", "dequant.cu", "batch.cu", "dynamic.cu", "layout.cu", "focus.cu", "gptq.cu"]
HEADERS = ["device.cuh", "launch.h", "screen.cuh", "nvfp4_block.cuh", "mxfp4_block.cuh", "batch.h", "wait.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfp4q.so")


def _inputs():
    return ([os.path.join(SRC, s) for s in SOURCES + HEADERS] +
            [os.path.join(ROOT, "include", "fp4q.h"), os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(os.path.join(HERE, "_build"), exist_ok=True)
    cmd = [nvcc_path(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "--fmad=false", "-Xptxas", "--fmad=false",
           "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
           "-I", os.path.join(ROOT, "include"),
           *[os.path.join(SRC, s) for s in SOURCES], "-o", LIB + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(HERE, "_build", "ptxas.log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libfp4q.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
