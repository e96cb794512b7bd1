"""Build libnvfp4trace.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m train_rollout_alignment_b200.build [--verbose]

FP32 arithmetic must be bit-exact IEEE round-to-nearest: no --use_fast_math,
and -fmad=false so no multiply is contracted into an FMA.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libnvfp4trace.so")
SOURCES = ["api.cu", "quantize.cu", "stats.cu", "sr_transpose.cu", "rht.cu", "noalloc.cu",
           "next_formats.cu", "producer.cu", "transport.cu", "moe_dispatch.cu", "measure.cu"]
HEADERS = ["nvfp4_device.cuh", "stats_device.cuh", "launch.h", "umma.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS + ["exports.map"]]
    files.append(os.path.join(ROOT, "include", "nvfp4_trace.h"))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include")]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES] + ["-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
