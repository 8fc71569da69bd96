"""Builds libfmoe.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfmoe.so")
# the same sources with FMOE_TRACE: the fused kernel records phase timestamps
LIB_TRACE = os.path.join(HERE, "libfmoe_trace.so")
SOURCES = ["fmoe_api.cu", "fmoe_decode.cu", "fmoe_repack.cu", "fmoe_static.cu", "fmoe_batched.cu", "fmoe_grouped_tc.cu",
           "fmoe_requant.cu"]
HEADERS = ["fmoe_internal.h"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "fmoe.h"))
    files.append(os.path.abspath(__file__))
    return files


def stale(trace: bool = False) -> bool:
    lib = LIB_TRACE if trace else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    lib = LIB_TRACE if trace else LIB
    if not force and not stale(trace):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["nvcc", *NVCC_FLAGS, *(["-DFMOE_TRACE"] if trace else []), "-shared", "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES], "-lcudart"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    trace = "--trace" in sys.argv
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, trace=trace))
