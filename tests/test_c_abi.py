"""The C ABI used from plain C programs (tests/c/*.c), built here with gcc
against include/opt2s.h and linked to libopt2s.so: no Python binding and no
PyTorch on the path.  The GPU program also links the CPU oracle (test
infrastructure) and compares the device results with it bit for bit."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path, src, extra=()):
    from elementwise_optimizer_b200 import _build as b
    b.build()
    exe = str(tmp_path / os.path.basename(src).replace(".c", ""))
    pkg = os.path.join(ROOT, "elementwise_optimizer_b200")
    cmd = ["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), "-o", exe, os.path.join(ROOT, "tests", "c", src),
           "-L", pkg, "-lopt2s", f"-Wl,-rpath,{pkg}", *extra]
    subprocess.run(cmd, check=True)
    return exe


def test_c_program_host_checks(tmp_path):
    exe = _build(tmp_path, "abi_host_check.c")
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


@pytest.mark.gpu
def test_c_program_steps_on_gpu_bitwise_equal_to_oracle(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    lib = oracle.build()
    exe = _build(tmp_path, "abi_gpu_step.c",
                 extra=[lib, f"-Wl,-rpath,{os.path.dirname(lib)}",
                        "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                        f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
