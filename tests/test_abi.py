"""CPU tests of the C ABI: the library loads, exports every declared symbol,
its structs match the header, and argument validation returns the documented
status codes before touching a GPU.  No compute call runs here.
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fused_linear.h")


@pytest.fixture(scope="module")
def fl():
    from gemm_bias_activation_tcgen05_b200 import build
    build.build()
    import gemm_bias_activation_tcgen05_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fl_[a-z_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ["fl_plan", "fl_execute", "fl_free", "fl_relu_backward", "fl_check_status", "fl_last_error"]:
        assert n in names


def test_library_exports_every_declared_symbol(fl):
    lib = ctypes.CDLL(fl.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(fl.EXPORTED) == declared_functions()


def test_struct_layout_matches_header(fl):
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "fused_linear.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(fl_epilogue_desc), offsetof(fl_epilogue_desc, scale),
         offsetof(fl_epilogue_desc, lda), offsetof(fl_epilogue_desc, unfused), sizeof(fl_plan_info),
         offsetof(fl_plan_info, launches_per_execute));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = list(map(int, subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()))
    E, I = fl.fl_epilogue_desc, fl.fl_plan_info
    assert vals == [ctypes.sizeof(E), E.scale.offset, E.lda.offset, E.unfused.offset, ctypes.sizeof(I),
                    I.launches_per_execute.offset]


def _plan_status(fl, M=256, N=256, K=64, dtype="bf16", compute="32F", **epi):
    e = fl.make_epilogue(**epi)
    h = ctypes.c_void_p()
    st = fl.LIB.fl_plan(ctypes.byref(h), M, N, K, fl.DTYPES[dtype], fl.COMPUTES[compute], ctypes.byref(e))
    return st, h


@pytest.mark.parametrize("args,status", [
    (dict(M=0), "FL_ERR_INVALID_ARG"),
    (dict(N=0), "FL_ERR_INVALID_ARG"),
    (dict(K=-1), "FL_ERR_INVALID_ARG"),
    (dict(dtype="f32", compute="32F"), "FL_ERR_UNSUPPORTED"),
    (dict(dtype="bf16", compute="32F_3XTF32"), "FL_ERR_UNSUPPORTED"),
    (dict(kind="GEGLU_TANH", b_major=1), "FL_ERR_UNSUPPORTED"),
    (dict(kind="GEGLU_TANH", out_dtype="f32"), "FL_ERR_UNSUPPORTED"),
    (dict(lda=60), "FL_ERR_INVALID_ARG"),          # smaller than K
    (dict(K=63, lda=0), "FL_ERR_ALIGNMENT"),        # 126-byte rows
    (dict(N=100, ldo=100, out_dtype="bf16"), "FL_ERR_ALIGNMENT"),
    (dict(bias_axis=2), "FL_ERR_INVALID_ARG"),
    (dict(b_major=3), "FL_ERR_INVALID_ARG"),
])
def test_plan_validation(fl, args, status):
    shape = {k: args.pop(k) for k in ("M", "N", "K", "dtype", "compute") if k in args}
    st, _ = _plan_status(fl, **shape, **args)
    assert fl.STATUS_NAMES[st] == status, fl.fl_last_error()
    assert fl.fl_last_error()


def test_plan_rejects_unknown_kind_and_reserved(fl):
    e = fl.make_epilogue()
    e.kind = 99
    h = ctypes.c_void_p()
    assert fl.LIB.fl_plan(ctypes.byref(h), 8, 8, 8, 1, 0, ctypes.byref(e)) == fl.FL_ERR_INVALID_ARG
    e = fl.make_epilogue()
    e.reserved[1] = 5
    assert fl.LIB.fl_plan(ctypes.byref(h), 8, 8, 8, 1, 0, ctypes.byref(e)) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_plan(None, 8, 8, 8, 1, 0, ctypes.byref(e)) == fl.FL_ERR_INVALID_ARG


def test_valid_plan_without_gpu_reports_device(fl):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st, h = _plan_status(fl, kind="GELU_BIAS")
    assert st == fl.FL_ERR_DEVICE
    assert h.value is None


def test_null_handles(fl):
    assert fl.LIB.fl_free(None) == fl.FL_OK
    assert fl.LIB.fl_execute(None, None, None, None, None, None, None, None) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_check_status(None, None) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_relu_backward(None, None, None, 4, 4, 0, 0, 1, None) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_get_plan_info(None, None) == fl.FL_ERR_INVALID_ARG
    with pytest.raises(fl.FusedLinearError):
        fl.fl_relu_backward(None, None, None, 4, 4, "bf16")


def test_relu_backward_validation(fl):
    # misaligned pointers and bad sizes are rejected before any launch
    assert fl.LIB.fl_relu_backward(2, 4, 2, 4, 4, 0, 0, 2, None) == fl.FL_ERR_ALIGNMENT
    assert fl.LIB.fl_relu_backward(16, 16, 16, -1, 4, 0, 0, 1, None) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_relu_backward(16, 16, 16, 4, 8, 4, 0, 1, None) == fl.FL_ERR_INVALID_ARG
    assert fl.LIB.fl_relu_backward(16, 16, 16, 4, 4, 0, 0, 7, None) == fl.FL_ERR_INVALID_ARG


def test_backward_and_layernorm_validation(fl):
    # every argument check runs before the first CUDA call, so it works without a GPU
    L = fl.LIB
    INV, ALN = fl.FL_ERR_INVALID_ARG, fl.FL_ERR_ALIGNMENT
    # fl_drelu_bgrad(grad, aux, dpre, dbias, M, N, ld_grad, ld_dpre, dtype, ws, ws_bytes, stream)
    assert L.fl_drelu_bgrad(None, 16, 16, None, 4, 4, 0, 0, 1, None, 0, None) == INV
    assert L.fl_drelu_bgrad(16, 16, 16, None, -1, 4, 0, 0, 1, None, 0, None) == INV
    assert L.fl_drelu_bgrad(16, 16, 16, None, 4, 8, 4, 0, 1, None, 0, None) == INV   # ld < N
    assert L.fl_drelu_bgrad(16, 16, 16, None, 4, 4, 0, 0, 9, None, 0, None) == INV   # dtype
    assert L.fl_drelu_bgrad(16, 18, 16, None, 4, 4, 0, 0, 1, None, 0, None) == ALN   # mask not 4-byte aligned
    # fl_dgelu_bgrad(grad, v, dpre, dbias, M, N, ld_grad, ld_v, ld_dpre, dtype, ws, ws_bytes, stream)
    assert L.fl_dgelu_bgrad(16, None, 16, None, 4, 4, 0, 0, 0, 1, None, 0, None) == INV
    assert L.fl_dgelu_bgrad(16, 17, 16, None, 4, 4, 0, 0, 0, 1, None, 0, None) == ALN
    assert L.fl_dgelu_bgrad(16, 16, 16, 18, 4, 4, 0, 0, 0, 1, None, 0, None) == ALN  # dbias not 4-byte aligned
    n = ctypes.c_size_t()
    assert L.fl_bias_grad_workspace_size(-1, 4, 1, ctypes.byref(n)) == INV
    assert L.fl_bias_grad_workspace_size(4, 4, 1, None) == INV
    # fl_layernorm(x, gamma, beta, z, M, N, ld_x, ld_z, x_dtype, z_dtype, param_dtype, eps, stream)
    assert L.fl_layernorm(None, None, None, 16, 4, 4, 0, 0, 2, 2, 2, 1e-5, None) == INV
    assert L.fl_layernorm(16, None, None, 16, 4, 4, 0, 0, 2, 2, 2, -1.0, None) == INV   # eps < 0
    assert L.fl_layernorm(16, None, None, 16, 4, 8, 4, 0, 2, 2, 2, 1e-5, None) == INV   # ld < N
    assert L.fl_layernorm(18, None, None, 16, 4, 4, 0, 0, 2, 2, 2, 1e-5, None) == ALN   # x not 4-byte aligned
    assert L.fl_layernorm(16, None, None, 16, 4, 4, 0, 0, 2, 2, 5, 1e-5, None) == INV   # param dtype
    assert L.fl_wait_selftest(0, None) == INV


SOURCES = [os.path.join(ROOT, "gemm_bias_activation_tcgen05_b200", "csrc", f)
           for f in ("fl_api.cu", "fl_gemm.cuh", "fl_ptx.cuh", "fl_elementwise.cuh")]


def test_no_multicast_load_anywhere():
    # No TMA or bulk load with cluster multicast in any source: the one use of the
    # qualifier allowed is a tcgen05.commit that arrives on the same barrier of both CTAs
    # of a pair.  (The qualifier is assembled here so that this file does not spell it out.)
    needle = ".multicast" + "::" + "cluster"
    for p in SOURCES + [HEADER]:
        for i, line in enumerate(open(p), 1):
            if needle in line:
                assert "tcgen05.commit" in line and "cp.async" not in line and "bulk" not in line, f"{p}:{i}"


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "gemm_bias_activation_tcgen05_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
                assert "oracle/" not in text, f
