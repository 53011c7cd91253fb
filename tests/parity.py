"""Shared helpers of the GPU parity tests: run one layer through the C ABI and
compare it with the oracle element by element.

Tolerances
  * the contract: 16-bit outputs |gpu − oracle| ≤ 2e-2·max(1, |oracle|);
    fp32 outputs ≤ 1e-3·max(1, |oracle|); the ReLU mask bit-exact wherever
    |pre-activation| > 1e-3.
  * a tighter check derived from the arithmetic, because the contract's
    absolute floor of 2e-2 is larger than the outputs of the N(0,1)/64
    workloads: max error ≤ 2 units in the last place of the output dtype at
    max|oracle| plus 2^-14·max_k-sum |a||w| (fp32 accumulation in a different
    order over K ≤ 4096 terms).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

import oracle

TD = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
ULP_REL = {"bf16": 2.0 ** -7, "f16": 2.0 ** -10, "f32": 2.0 ** -23}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def contract_tol(o: np.ndarray, out_dtype: str) -> np.ndarray:
    c = 1e-3 if out_dtype == "f32" else 2e-2
    return c * np.maximum(1.0, np.abs(o))


def check_close(got: np.ndarray, ref: np.ndarray, out_dtype: str, absdot_max: float, what: str = ""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = contract_tol(ref, out_dtype)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} elements outside the contract tolerance; "
                           f"worst {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")
    tight = 2.0 * ULP_REL[out_dtype] * float(np.abs(ref).max()) + 2.0 ** -14 * absdot_max + 1e-30
    assert err.max() <= tight, f"{what}: max error {err.max():.3e} above the arithmetic bound {tight:.3e}"
    return float(err.max())


def check_mask(aux_gpu: np.ndarray, v: np.ndarray, N: int, what: str = "", margin=None):
    """Bits must equal (v > 0) wherever |v| > 1e-3 (+ margin); padding bits must be 0.

    ``margin`` widens the undecided band for a path that rounds an intermediate
    (the unfused twin stores A·Wᵀ in the output dtype before adding the bias).
    """
    M = v.shape[0]
    words = (N + 31) // 32
    assert aux_gpu.shape == (M, words)
    a = aux_gpu.astype(np.uint64)
    bits = np.zeros((M, words * 32), dtype=bool)
    for j in range(32):
        bits[:, j::32] = ((a >> np.uint64(j)) & np.uint64(1)).astype(bool)
    assert not bits[:, N:].any(), f"{what}: padding bits set"
    bits = bits[:, :N]
    decided = np.abs(v) > 1e-3 + (0.0 if margin is None else margin)
    mism = (bits != (v > 0)) & decided
    assert not mism.any(), f"{what}: {mism.sum()} mask bits differ where |v| > 1e-3"


def poison(shape, dtype: str, device="cuda") -> torch.Tensor:
    return torch.full(shape, float("nan"), dtype=TD[dtype], device=device)


def run_linear(fl, *, M, N, K, dtype, epilogue, out_dtype, A, W, bias=None, bias_dtype="bf16",
               bias_axis=0, b_major=0, residual=None, residual_dtype="bf16", scale=1.0,
               unfused=False, out_pad=8, stream=None, check_canary=True, schedule="auto",
               bias_offset=0) -> Dict[str, np.ndarray]:
    """Run one layer; A/W/bias/residual are CPU tensors in (padded) storage.

    bias_offset > 0 places the bias that many elements into its device buffer (a pointer
    off the 16-byte grid for odd offsets).

    Returns the logical [M, N] output and the aux mask as numpy arrays.
    """
    dev = "cuda"
    dA, dW = A.to(dev), W.to(dev)
    dB = None
    if bias is not None:
        buf = torch.zeros(bias.numel() + bias_offset, dtype=bias.dtype, device=dev)
        dB = buf[bias_offset:]
        dB.copy_(bias.to(dev))
    dR = residual.to(dev) if residual is not None else None
    ldo = -(-N // out_pad) * out_pad
    out = poison((M, ldo), out_dtype)
    aux = None
    if epilogue == "RELU_AUX_BIAS":
        aux = torch.full((M, (N + 31) // 32), -559038737, dtype=torch.int32, device=dev)  # 0xDEADBEEF
    plan = fl.Plan(M, N, K, dtype=dtype, compute="32F_3XTF32" if dtype == "f32" else "32F",
                   kind=epilogue, out_dtype=out_dtype, bias_dtype=bias_dtype,
                   residual_dtype=residual_dtype, bias_axis=bias_axis,
                   has_residual=residual is not None, scale=scale, b_major=b_major,
                   lda=A.shape[1], ldb=W.shape[1], ldo=ldo,
                   ldr=residual.shape[1] if residual is not None else 0, unfused=unfused, schedule=schedule)
    try:
        plan.execute(dA, dW, dB, aux, dR, out, stream)
        st = plan.check(stream)
        assert st == fl.FL_OK, f"status {fl.STATUS_NAMES.get(st)}: {fl.fl_last_error()}"
        info = plan.info()
    finally:
        plan.free()
    res = {"out": to64(out[:, :N]), "info": info}
    if check_canary and ldo > N:
        pad = out[:, N:].float()
        assert torch.isnan(pad).all(), "kernel wrote into the padding of the output rows"
    if aux is not None:
        res["aux"] = aux.cpu().numpy().view(np.uint32)
    return res


def oracle_linear(*, A, W, bias=None, bias_axis=0, b_major=0, residual=None, scale=1.0, epilogue,
                  out_dtype, M, N, K, rows=None):
    """Oracle on the logical extents (rows: optional subset of output rows)."""
    a = to64(A)[:, :K]
    w = to64(W)[:K, :N] if b_major else to64(W)[:N, :K]
    r = to64(residual)[:, :N] if residual is not None else None
    b = to64(bias) if bias is not None else None
    if rows is not None:
        a = a[rows]
        r = r[rows] if r is not None else None
        if b is not None and bias_axis == 1:
            b = b[rows]
    y, aux, v = oracle.fused_linear(a, w, b, epilogue=epilogue, out_dtype=out_dtype, bias_axis=bias_axis,
                                    b_major=b_major, residual=r, scale=scale)
    absdot = oracle.gemm(np.abs(a), np.abs(w), b_major)
    return y, aux, v, float(absdot.max()) if absdot.size else 0.0


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    r = np.random.default_rng(seed)
    rows = set([0, M - 1, min(M - 1, 127), min(M - 1, 128)])
    rows.update(r.choice(M, size=min(n, M), replace=False).tolist())
    return np.array(sorted(rows))
