"""Builds libopt2s.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m elementwise_optimizer_b200._build [--verbose]

The device code is compiled with IEEE division and square root, no
flush-to-zero and no FMA contraction (the kernel also spells every operation
as an explicit round-to-nearest intrinsic), so its arithmetic matches the
documented fp32 operation order exactly.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libopt2s.so")

SOURCES = [os.path.join(CSRC, "opt2s_kernel.cu"), os.path.join(CSRC, "opt2s_kernel8.cu"),
           os.path.join(CSRC, "opt2s_api.cpp"), os.path.join(CSRC, "opt2s_api8.cpp"),
           os.path.join(CSRC, "opt2s_noalloc.cu")]
HEADERS = [os.path.join(CSRC, "opt2s_internal.h"), os.path.join(CSRC, "opt2s_device.cuh"),
           os.path.join(INCLUDE, "opt2s.h"), os.path.join(INCLUDE, "opt2s_testing.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared",
         "-Xcompiler", "-fPIC,-fvisibility=hidden,-O2",
         "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-fmad=false",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-Xptxas", "-v"] if verbose else []),
           "-o", tmp, *SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
