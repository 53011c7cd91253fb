"""The C ABI from a plain C99 program (no Python, no CUDA headers), on the CPU.

tests/c/abi_client.c includes only include/fused_linear.h, is compiled by gcc with
-std=c99 -Wall -Wextra -Werror and linked against the built libfused_linear.so, then run:
it previews two configurations and checks that bad arguments return status codes with a
message.  Skipped when gcc or the library is missing.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "gemm_bias_activation_tcgen05_b200")


def test_c_client_builds_and_runs(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None or not os.path.exists(os.path.join(LIBDIR, "libfused_linear.so")):
        pytest.skip("needs gcc and the built library")
    exe = tmp_path / "abi_client"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_client.c"), "-L", LIBDIR, "-lfused_linear",
                    f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 failure(s)" in r.stdout


def test_kernel_schedule_on_the_host(tmp_path):
    """The kernel's own stream-K schedule function, compiled for the host by nvcc
    (tests/c/schedule_check.cu): every (tile, K block) unit computed once, one finisher
    per cut tile, whose writer list is exactly the clusters that store a partial."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("needs nvcc")
    exe = tmp_path / "schedule_check"
    r = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                        os.path.join(ROOT, "tests", "c", "schedule_check.cu"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "schedule ok" in r.stdout
