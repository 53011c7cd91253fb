"""Build the sm_100a shared library ``libfused_linear.so`` in-tree with nvcc.

The library holds the C ABI of ``include/fused_linear.h`` and every CUDA
kernel of the fused linear layer.  It links the CUDA runtime statically and
reaches the driver's tensor-map encoder through the runtime's driver entry
point, so loading it needs no libcuda at link time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfused_linear.so")
SOURCES = [os.path.join(HERE, "csrc", "fl_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in ("fl_gemm.cuh", "fl_ptx.cuh", "fl_elementwise.cuh")] + \
    [os.path.join(ROOT, "include", "fused_linear.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(extra=()):
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
            "--shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-Xptxas", "-v",
            f"-I{os.path.join(ROOT, 'include')}", *extra, *SOURCES, "-o", LIB]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = command()
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libfused_linear.so")
    with open(os.path.join(HERE, "ptxas_report.txt"), "w") as f:
        f.write(r.stderr)
    if verbose:
        sys.stderr.write(r.stderr)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
