"""Builds the C-ABI library in-tree with nvcc for sm_100a.

    python -m elementwise_optimizer_b200._build [--verbose] [--nvtx]

Two shared libraries come out of one set of compiled objects:
  libopt2s.so          the product: every entry point of include/opt2s.h
                       and the read-only introspection of opt2s_testing.h;
  libopt2s_testing.so  the same objects (the same kernels) plus the forcing
                       knobs, the fault injection and the division check of
                       opt2s_testing.h, which the tests use to vary the launch
                       geometry and to make failures on the host.  Only the
                       host API translation unit is compiled twice.

The device code is compiled with IEEE division and square root, no
flush-to-zero and no FMA contraction (the kernels also spell every operation
as an explicit round-to-nearest intrinsic), so its arithmetic matches the
documented fp32 operation order exactly.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libopt2s.so")
TESTING_LIB = os.path.join(PKG, "libopt2s_testing.so")
# the optimizer front end's marshalling helper (a PyTorch C++ extension)
MARSHAL_SRC = os.path.join(PKG, "csrc", "opt2s_marshal.cpp")
MARSHAL_DIR = os.path.join(PKG, "_build")
MARSHAL_NAME = "opt2s_marshal"

COMMON = ["opt2s_kernel.cu", "opt2s_kernel8.cu", "opt2s_noalloc.cu", "opt2s_api8.cpp", "opt2s_ipc.cpp"]
API = "opt2s_api.cpp"
TESTING_ONLY = ["opt2s_testing.cu"]
SOURCES = [os.path.join(CSRC, f) for f in COMMON + [API] + TESTING_ONLY]
HEADERS = [os.path.join(CSRC, "opt2s_internal.h"), os.path.join(CSRC, "opt2s_device.cuh"),
           os.path.join(INCLUDE, "opt2s.h"), os.path.join(INCLUDE, "opt2s_testing.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC,-fvisibility=hidden,-O2",
         "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-fmad=false",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(marshal_path()) or os.path.getmtime(marshal_path()) < os.path.getmtime(MARSHAL_SRC):
        return True
    for lib in (LIB, TESTING_LIB):
        if not os.path.exists(lib):
            return True
        t = os.path.getmtime(lib)
        if any(os.path.getmtime(f) > t for f in SOURCES + HEADERS):
            return True
    return False


def marshal_path() -> str:
    return os.path.join(MARSHAL_DIR, MARSHAL_NAME + ".so")


def build_marshal(force: bool = False, verbose: bool = False) -> str:
    """Compile the optimizer's marshalling extension in-tree (host C++ against
    PyTorch's headers; no device code)."""
    out = marshal_path()
    header = os.path.join(INCLUDE, "opt2s.h")
    if (not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(MARSHAL_SRC)
            and os.path.getmtime(out) >= os.path.getmtime(header)):
        return out
    os.makedirs(MARSHAL_DIR, exist_ok=True)
    from torch.utils import cpp_extension
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    cpp_extension.load(name=MARSHAL_NAME, sources=[MARSHAL_SRC], build_directory=MARSHAL_DIR,
                       extra_cflags=["-O2"], extra_include_paths=[INCLUDE, cuda_inc], verbose=verbose)
    return out


def build(force: bool = False, verbose: bool = False, nvtx: bool = False) -> str:
    """Compile and link both libraries (if missing or older than a source).
    nvtx: wrap each step entry point in an NVTX range (OPT2S_NVTX=1 in the
    environment does the same).  Returns the product library's path."""
    nvtx = nvtx or os.environ.get("OPT2S_NVTX", "") not in ("", "0")
    if not force and not stale():
        return LIB
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DOPT2S_NVTX"] if nvtx else [])
    with tempfile.TemporaryDirectory() as tmp:
        jobs = [(f, os.path.join(tmp, f + ".o"), []) for f in COMMON + TESTING_ONLY]
        jobs += [(API, os.path.join(tmp, "api_product.o"), []),
                 (API, os.path.join(tmp, "api_testing.o"), ["-DOPT2S_TESTING"])]

        def compile_one(job):
            src, obj, defs = job
            r = subprocess.run([nvcc(), *ARCH, *FLAGS, *extra, *defs, "-c", "-o", obj,
                                os.path.join(CSRC, src)], capture_output=True, text=True)
            return src, r

        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
            for src, r in ex.map(compile_one, jobs):
                if verbose or r.returncode != 0:
                    sys.stderr.write(r.stdout + r.stderr)
                if r.returncode != 0:
                    raise subprocess.CalledProcessError(r.returncode, f"nvcc {src}")
        common = [os.path.join(tmp, f + ".o") for f in COMMON]
        links = [(LIB, common + [os.path.join(tmp, "api_product.o")]),
                 (TESTING_LIB, common + [os.path.join(tmp, "api_testing.o")] +
                  [os.path.join(tmp, f + ".o") for f in TESTING_ONLY])]
        for out, objs in links:
            subprocess.run([nvcc(), *ARCH, "-shared", "-o", out + ".tmp", *objs], check=True)
            os.replace(out + ".tmp", out)
    build_marshal(force=force, verbose=verbose)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv, nvtx="--nvtx" in sys.argv)
    print(LIB)
    print(TESTING_LIB)
