"""The allocation-free entry point against the planned one (GPU).

fl_execute_noalloc serves callers that cannot call cudaMalloc (a host whose
own pool owns all device memory, or a latency-critical path where allocation
and its possible device synchronisation are forbidden).  Its scratch lives in
a fixed device array inside the library and is shared by every call, so this
file makes two calls in a row on the same array and compares both with
fl_plan/fl_execute on the same inputs and with the oracle, within the parity
tests' tolerance (the ReLU mask bit-exact where the pre-activation is decided).
It is collected last and runs alone or after the other tests.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import gemm_bias_activation_tcgen05_b200 as m
    return m


CASES = [
    # (M, N, K, kind, out_dtype, residual, unfused)
    (256, 384, 192, "RELU_AUX_BIAS", "bf16", False, True),   # intermediate in the fixed scratch
    (200, 264, 128, "GELU_BIAS", "f32", True, True),
    (300, 520, 200, "GELU_TANH_BIAS", "bf16", False, False),  # fused: scratch is the error word only
]


def _run(fl, noalloc, M, N, K, kind, out_dtype, residual, unfused, seed):
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", seed, bias_dtype="bf16", residual=residual)
    dev = {k: v.cuda() for k, v in inp.items()}
    out = P.poison((M, N), out_dtype)
    aux = (torch.full((M, (N + 31) // 32), -1, dtype=torch.int32, device="cuda")
           if kind == "RELU_AUX_BIAS" else None)
    epi = fl.make_epilogue(kind=kind, out_dtype=out_dtype, bias_dtype="bf16", residual_dtype="bf16",
                           has_residual=residual, scale=0.5 if residual else 1.0, lda=inp["A"].shape[1],
                           ldb=inp["W"].shape[1], ldr=inp["residual"].shape[1] if residual else 0,
                           unfused=unfused)
    if noalloc:
        # straight through the C ABI
        st = fl.LIB.fl_execute_noalloc(M, N, K, fl.FL_BF16, fl.FL_COMPUTE_32F, ctypes.byref(epi),
                                       dev["A"].data_ptr(), dev["W"].data_ptr(), dev["bias"].data_ptr(),
                                       aux.data_ptr() if aux is not None else None,
                                       dev["residual"].data_ptr() if residual else None, out.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
        assert st == fl.FL_OK, fl.fl_last_error()
    else:
        h = fl.fl_plan(M, N, K, "bf16", "32F", epi)
        try:
            fl.fl_execute(h, dev["A"], dev["W"], dev["bias"], aux, dev.get("residual"), out)
            assert fl.fl_check_status(h) == fl.FL_OK, fl.fl_last_error()
        finally:
            fl.fl_free(h)
    torch.cuda.synchronize()
    return inp, P.to64(out), (aux.cpu().numpy().view(np.uint32) if aux is not None else None)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[3]}-{c[4]}-{'unfused' if c[6] else 'fused'}")
def test_noalloc_matches_planned_entry_point_twice(fl, case):
    M, N, K, kind, out_dtype, residual, unfused = case
    inp, ref, ref_aux = _run(fl, False, *case, seed=31)
    y, _, v, absdot = P.oracle_linear(A=inp["A"], W=inp["W"], bias=inp["bias"], residual=inp.get("residual"),
                                      scale=0.5 if residual else 1.0, epilogue=kind, out_dtype=out_dtype,
                                      M=M, N=N, K=K)
    # the unfused path rounds acc = A·Wᵀ to the output type before its bias step
    acc = v - P.to64(inp["bias"])[None, :]
    margin = P.ULP_REL[out_dtype] * (np.abs(acc) + np.abs(v)) if unfused else None
    for call in range(2):  # the second call finds the first call's scratch contents
        _, got, got_aux = _run(fl, True, *case, seed=31)
        P.check_close(got, ref, out_dtype, absdot, f"noalloc call {call} {kind} vs fl_execute")
        P.check_close(got, y, out_dtype, absdot, f"noalloc call {call} {kind} vs oracle")
        if ref_aux is not None:
            assert np.array_equal(got_aux, ref_aux)
            P.check_mask(got_aux, v, N, f"noalloc call {call} mask vs oracle", margin)


def test_noalloc_rejects_oversized_scratch(fl):
    # the unfused intermediate of 8192 x 4096 bf16 (64 MiB) does not fit the 32 MiB array
    epi = fl.make_epilogue(kind="BIAS", out_dtype="bf16", unfused=True)
    st = fl.LIB.fl_execute_noalloc(8192, 4096, 64, fl.FL_BF16, fl.FL_COMPUTE_32F, ctypes.byref(epi),
                                   16, 16, 16, None, None, 16, None)
    assert st == fl.FL_ERR_INVALID_ARG
    assert "scratch" in fl.fl_last_error()
