"""Python binding of the B200 fused linear layer (``include/fused_linear.h``).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libfused_linear.so``.  Tensors are passed by device pointer; the binding
never computes anything itself and has no CPU fallback — importing it without
the built library raises, and every call that launches work fails loudly
without a B200.

The entry points keep the C names: ``fl_plan``, ``fl_execute``, ``fl_free``,
``fl_relu_backward``, ``fl_check_status``, ``fl_get_plan_info``,
``fl_last_error``, ``fl_set_wait_limit_ns``, ``fl_execute_noalloc``, ``fl_bias_grad_workspace_size``,
``fl_drelu_bgrad``, ``fl_dgelu_bgrad``, ``fl_layernorm``, ``fl_wait_selftest``, ``fl_plan_preview``.
``Plan`` is a small owner of one plan handle (the cuBLASLt epilog page's Matmul → plan → execute → free).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfused_linear.so")

# ---------------------------------------------------------------- enums (mirror the header)
FL_OK, FL_ERR_INVALID_ARG, FL_ERR_UNSUPPORTED, FL_ERR_ALIGNMENT, FL_ERR_CUDA, FL_ERR_OOM, \
    FL_ERR_TIMEOUT, FL_ERR_DEVICE = range(8)
STATUS_NAMES = {0: "FL_OK", 1: "FL_ERR_INVALID_ARG", 2: "FL_ERR_UNSUPPORTED", 3: "FL_ERR_ALIGNMENT",
                4: "FL_ERR_CUDA", 5: "FL_ERR_OOM", 6: "FL_ERR_TIMEOUT", 7: "FL_ERR_DEVICE"}
FL_F16, FL_BF16, FL_F32 = 0, 1, 2
FL_COMPUTE_32F, FL_COMPUTE_32F_3XTF32 = 0, 1
EPILOGUES = {"NONE": 0, "BIAS": 1, "RELU_BIAS": 2, "RELU_AUX_BIAS": 3, "GELU_BIAS": 4,
             "GELU_TANH_BIAS": 5, "GEGLU_TANH": 6, "GELU_AUX_BIAS": 7,
             "GELU_SIGMOID_BIAS": 8}
DTYPES = {"f16": FL_F16, "bf16": FL_BF16, "f32": FL_F32}
COMPUTES = {"32F": FL_COMPUTE_32F, "32F_3XTF32": FL_COMPUTE_32F_3XTF32}
SCHEDULES = {"auto": 0, "data_parallel": 1, "stream_k": 2}

EXPORTED = ["fl_plan", "fl_execute", "fl_relu_backward", "fl_check_status", "fl_get_plan_info",
            "fl_free", "fl_last_error", "fl_set_wait_limit_ns", "fl_execute_noalloc",
            "fl_bias_grad_workspace_size", "fl_drelu_bgrad", "fl_dgelu_bgrad", "fl_layernorm", "fl_wait_selftest",
            "fl_plan_preview"]


class fl_epilogue_desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("out_dtype", ctypes.c_int32), ("bias_dtype", ctypes.c_int32),
                ("residual_dtype", ctypes.c_int32), ("bias_axis", ctypes.c_int32),
                ("has_residual", ctypes.c_int32), ("scale", ctypes.c_float), ("b_major", ctypes.c_int32),
                ("lda", ctypes.c_int64), ("ldb", ctypes.c_int64), ("ldo", ctypes.c_int64),
                ("ldr", ctypes.c_int64), ("unfused", ctypes.c_int32), ("schedule", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class fl_plan_info(ctypes.Structure):
    _fields_ = [("tile_m", ctypes.c_int32), ("tile_n", ctypes.c_int32), ("mma_n", ctypes.c_int32),
                ("swap_ab", ctypes.c_int32), ("split_k", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("smem_bytes", ctypes.c_int32),
                ("launches_per_execute", ctypes.c_int32), ("cta_pair", ctypes.c_int32),
                ("stream_k_tiles", ctypes.c_int32), ("stream_k_pairs", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 4)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libfused_linear.so is not built ({LIB_PATH}); run "
            "`python gemm_bias_activation_tcgen05_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.fl_plan.argtypes = [ctypes.POINTER(vp), i64, i64, i64, i32, i32, ctypes.POINTER(fl_epilogue_desc)]
    lib.fl_plan.restype = i32
    lib.fl_execute.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    lib.fl_execute.restype = i32
    lib.fl_relu_backward.argtypes = [vp, vp, vp, i64, i64, i64, i64, i32, vp]
    lib.fl_relu_backward.restype = i32
    lib.fl_check_status.argtypes = [vp, vp]
    lib.fl_check_status.restype = i32
    lib.fl_get_plan_info.argtypes = [vp, ctypes.POINTER(fl_plan_info)]
    lib.fl_get_plan_info.restype = i32
    lib.fl_plan_preview.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(fl_epilogue_desc), i32, i32,
                                    ctypes.POINTER(fl_plan_info)]
    lib.fl_plan_preview.restype = i32
    lib.fl_free.argtypes = [vp]
    lib.fl_free.restype = i32
    lib.fl_last_error.argtypes = []
    lib.fl_last_error.restype = ctypes.c_char_p
    lib.fl_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.fl_set_wait_limit_ns.restype = i32
    lib.fl_execute_noalloc.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(fl_epilogue_desc),
                                       vp, vp, vp, vp, vp, vp, vp]
    lib.fl_execute_noalloc.restype = i32
    lib.fl_bias_grad_workspace_size.argtypes = [i64, i64, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.fl_bias_grad_workspace_size.restype = i32
    lib.fl_drelu_bgrad.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i32, vp, ctypes.c_size_t, vp]
    lib.fl_drelu_bgrad.restype = i32
    lib.fl_dgelu_bgrad.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, vp, ctypes.c_size_t, vp]
    lib.fl_dgelu_bgrad.restype = i32
    lib.fl_layernorm.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i32, i32, i32, ctypes.c_float, vp]
    lib.fl_layernorm.restype = i32
    lib.fl_wait_selftest.argtypes = [ctypes.c_uint64, vp]
    lib.fl_wait_selftest.restype = i32
    return lib


LIB = _load()


class FusedLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = LIB.fl_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def _check(st: int, where: str) -> None:
    if st != FL_OK:
        raise FusedLinearError(st, where)


def _ptr(x) -> Optional[int]:
    """Device address of a tensor (or an int address); None stays NULL."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- C names
def fl_last_error() -> str:
    return LIB.fl_last_error().decode(errors="replace")


def fl_set_wait_limit_ns(ns: int) -> None:
    _check(LIB.fl_set_wait_limit_ns(int(ns)), "fl_set_wait_limit_ns")


def make_epilogue(kind: str = "NONE", out_dtype: str = "bf16", bias_dtype: str = "bf16",
                  residual_dtype: str = "bf16", bias_axis: int = 0, has_residual: bool = False,
                  scale: float = 1.0, b_major: int = 0, lda: int = 0, ldb: int = 0, ldo: int = 0,
                  ldr: int = 0, unfused: bool = False, schedule: str = "auto") -> fl_epilogue_desc:
    e = fl_epilogue_desc()
    e.kind = EPILOGUES[kind]
    e.out_dtype = DTYPES[out_dtype]
    e.bias_dtype = DTYPES[bias_dtype]
    e.residual_dtype = DTYPES[residual_dtype]
    e.bias_axis = int(bias_axis)
    e.has_residual = int(bool(has_residual))
    e.scale = float(scale)
    e.b_major = int(b_major)
    e.lda, e.ldb, e.ldo, e.ldr = int(lda), int(ldb), int(ldo), int(ldr)
    e.unfused = int(bool(unfused))
    e.schedule = SCHEDULES[schedule]
    return e


def fl_plan(M: int, N: int, K: int, dtype: str, compute: str, epi: fl_epilogue_desc) -> int:
    h = ctypes.c_void_p()
    _check(LIB.fl_plan(ctypes.byref(h), int(M), int(N), int(K), DTYPES[dtype], COMPUTES[compute],
                       ctypes.byref(epi)), "fl_plan")
    return h.value


def fl_execute(plan: int, A, W, bias=None, aux=None, residual=None, out=None, stream=None) -> None:
    _check(LIB.fl_execute(plan, _ptr(A), _ptr(W), _ptr(bias), _ptr(aux), _ptr(residual), _ptr(out),
                          _stream(stream)), "fl_execute")


def fl_execute_noalloc(M: int, N: int, K: int, dtype: str, compute: str, epi: fl_epilogue_desc, A, W, bias=None,
                       aux=None, residual=None, out=None, stream=None) -> None:
    """One layer without device allocation: scratch comes from the library's fixed
    device array (for callers that cannot allocate; see the header)."""
    _check(LIB.fl_execute_noalloc(int(M), int(N), int(K), DTYPES[dtype], COMPUTES[compute], ctypes.byref(epi),
                                  _ptr(A), _ptr(W), _ptr(bias), _ptr(aux), _ptr(residual), _ptr(out),
                                  _stream(stream)), "fl_execute_noalloc")


def fl_relu_backward(grad, aux, dpre, M: int, N: int, dtype: str, ld_grad: int = 0, ld_dpre: int = 0,
                     stream=None) -> None:
    _check(LIB.fl_relu_backward(_ptr(grad), _ptr(aux), _ptr(dpre), int(M), int(N), int(ld_grad),
                                int(ld_dpre), DTYPES[dtype], _stream(stream)), "fl_relu_backward")


def fl_bias_grad_workspace_size(M: int, N: int, dtype: str) -> int:
    n = ctypes.c_size_t()
    _check(LIB.fl_bias_grad_workspace_size(int(M), int(N), DTYPES[dtype], ctypes.byref(n)),
           "fl_bias_grad_workspace_size")
    return int(n.value)


def fl_drelu_bgrad(grad, aux, dpre, dbias, M: int, N: int, dtype: str, workspace=None, workspace_bytes: int = 0,
                   ld_grad: int = 0, ld_dpre: int = 0, stream=None) -> None:
    _check(LIB.fl_drelu_bgrad(_ptr(grad), _ptr(aux), _ptr(dpre), _ptr(dbias), int(M), int(N), int(ld_grad),
                              int(ld_dpre), DTYPES[dtype], _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "fl_drelu_bgrad")


def fl_dgelu_bgrad(grad, v, dpre, dbias, M: int, N: int, dtype: str, workspace=None, workspace_bytes: int = 0,
                   ld_grad: int = 0, ld_v: int = 0, ld_dpre: int = 0, stream=None) -> None:
    _check(LIB.fl_dgelu_bgrad(_ptr(grad), _ptr(v), _ptr(dpre), _ptr(dbias), int(M), int(N), int(ld_grad),
                              int(ld_v), int(ld_dpre), DTYPES[dtype], _ptr(workspace), int(workspace_bytes),
                              _stream(stream)), "fl_dgelu_bgrad")


def fl_layernorm(x, gamma, beta, z, M: int, N: int, x_dtype: str, z_dtype: str, param_dtype: str = "f32",
                 eps: float = 1e-12, ld_x: int = 0, ld_z: int = 0, stream=None) -> None:
    _check(LIB.fl_layernorm(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(z), int(M), int(N), int(ld_x), int(ld_z),
                            DTYPES[x_dtype], DTYPES[z_dtype], DTYPES[param_dtype], float(eps), _stream(stream)),
           "fl_layernorm")


def fl_wait_selftest(limit_ns: int, stream=None) -> int:
    """Status of the bounded-wait failure-path self-test (FL_ERR_TIMEOUT when it works)."""
    return LIB.fl_wait_selftest(int(limit_ns), _stream(stream))


def fl_check_status(plan: int, stream=None) -> int:
    return LIB.fl_check_status(plan, _stream(stream))


def fl_get_plan_info(plan: int) -> dict:
    info = fl_plan_info()
    _check(LIB.fl_get_plan_info(plan, ctypes.byref(info)), "fl_get_plan_info")
    return {k: getattr(info, k) for k, _ in fl_plan_info._fields_ if k != "reserved"}


def fl_plan_preview(M: int, N: int, K: int, dtype: str = "bf16", compute: str = "32F", *, num_sms: int = 148,
                    max_smem_per_block: int = 232448, **epi) -> dict:
    """The configuration fl_plan would choose on a device with `num_sms` SMs and that much
    opt-in shared memory per block, computed on the host (no device needed)."""
    info = fl_plan_info()
    e = make_epilogue(**epi)
    _check(LIB.fl_plan_preview(int(M), int(N), int(K), DTYPES[dtype], COMPUTES[compute], ctypes.byref(e),
                               int(num_sms), int(max_smem_per_block), ctypes.byref(info)), "fl_plan_preview")
    return {k: getattr(info, k) for k, _ in fl_plan_info._fields_ if k != "reserved"}


def fl_free(plan: Optional[int]) -> None:
    _check(LIB.fl_free(plan), "fl_free")


class Plan:
    """Owner of one ``fl_plan_t``: plan at construction, ``execute`` per call, ``free`` at the end."""

    def __init__(self, M: int, N: int, K: int, dtype: str = "bf16", compute: str = "32F", **epi):
        self.M, self.N, self.K = M, N, K
        self.epi = make_epilogue(**epi)
        self.handle = fl_plan(M, N, K, dtype, compute, self.epi)

    def execute(self, A, W, bias=None, aux=None, residual=None, out=None, stream=None) -> None:
        fl_execute(self.handle, A, W, bias, aux, residual, out, stream)

    def info(self) -> dict:
        return fl_get_plan_info(self.handle)

    def check(self, stream=None) -> int:
        return fl_check_status(self.handle, stream)

    def free(self) -> None:
        if self.handle:
            fl_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass
