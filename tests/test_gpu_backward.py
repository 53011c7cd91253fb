"""GPU parity of the backward of the fused layer and of the GELU_AUX_BIAS forward.

dReLU with the bias gradient, GELU' from the stored pre-activation, against the
fp64 oracle.  Tolerances:
  * dReLU's dpre is bit-exact (grad times 0 or 1); GELU's dpre within one unit in
    the last place of its type (at least the subnormal quantum) plus the kernel's
    GELU' error (4e-7·|grad|).
  * dbias (fp32 sums in a fixed order) within 2^-24·(M + 16)·Σ_m|dpre| — the bound of
    a sequential fp32 sum of M terms — plus 4e-7·Σ_m|grad| for GELU'.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

GELU_GRAD_ABS = 4e-7  # bound on |GELU'(v) in fp32 - GELU'(v)| (erf to ~2e-7, e^(-v²/2) to ~2^-22)
# one unit in the last place at the bottom of each type's range (the subnormal quantum):
# there a rounding of a value within GELU_GRAD_ABS of a midpoint moves by this much
ULP_MIN = {"f16": 2.0 ** -24, "bf16": 2.0 ** -133, "f32": 2.0 ** -149}


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import gemm_bias_activation_tcgen05_b200 as m
    return m


def _workspace(fl, M, N, dtype):
    n = fl.fl_bias_grad_workspace_size(M, N, dtype)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device="cuda"), n


def _check_dbias(got, want_exact, abs_terms, M, grad_abs=None, what=""):
    tol = 2.0 ** -24 * (M + 16) * abs_terms + 1e-30
    if grad_abs is not None:
        tol = tol + GELU_GRAD_ABS * grad_abs
    err = np.abs(got - want_exact)
    assert np.all(err <= tol), f"{what}: dbias error {err.max():.3e} above its bound at {err.argmax()}"


def _grad(M, N, dtype, seed, ld=None):
    g = torch.Generator().manual_seed(seed)
    ld = ld or N
    return torch.randn(M, ld, generator=g, dtype=torch.float32).to(P.TD[dtype])


@pytest.mark.parametrize("M,N,dtype", [(300, 520, "bf16"), (257, 77, "f16"), (64, 1000, "f32"), (5, 4096, "bf16"),
                                       (1000, 24, "bf16")])
def test_drelu_bgrad(fl, M, N, dtype):
    g = torch.Generator().manual_seed(M + N)
    v = torch.randn(M, N, generator=g, dtype=torch.float64).numpy()
    v[0, :5] = 0.0  # ReLU'(0) = 0
    mask = oracle.relu_aux_mask(v)
    grad = _grad(M, N, dtype, M * 7 + N)
    dmask = torch.from_numpy(mask.view(np.int32)).cuda()
    dgrad = grad.cuda()
    dpre = P.poison((M, N), dtype)
    dbias = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    ws, nbytes = _workspace(fl, M, N, dtype)
    for rep in range(2):  # the workspace is left ready for the next call
        fl.fl_drelu_bgrad(dgrad, dmask, dpre, dbias, M, N, dtype, ws, nbytes)
        torch.cuda.synchronize()
        dv, db = oracle.drelu_bgrad(P.to64(grad), mask, N, dtype)
        assert np.array_equal(P.to64(dpre), dv), f"dpre differs (launch {rep})"
        _check_dbias(P.to64(dbias), db, np.abs(dv).sum(axis=0), M, what=f"drelu_bgrad {M}x{N} {dtype} launch {rep}")


def test_drelu_bgrad_without_bias_grad_and_aliasing(fl):
    M, N = 130, 300
    g = torch.Generator().manual_seed(3)
    v = torch.randn(M, N, generator=g, dtype=torch.float64).numpy()
    mask = oracle.relu_aux_mask(v)
    grad = _grad(M, N, "bf16", 4)
    buf = grad.cuda()
    fl.fl_drelu_bgrad(buf, torch.from_numpy(mask.view(np.int32)).cuda(), buf, None, M, N, "bf16")  # dpre = grad
    torch.cuda.synchronize()
    assert np.array_equal(P.to64(buf), oracle.drelu(P.to64(grad), mask, N, "bf16"))


def test_relu_aux_4096_backward_with_bias_grad(fl):
    w = workloads.get("relu_aux_4096")
    M, N = w.M, w.N
    g = torch.Generator().manual_seed(11)
    v = torch.randn(M, N, generator=g, dtype=torch.float32).numpy().astype(np.float64)
    mask = oracle.relu_aux_mask(v)
    grad = _grad(M, N, "bf16", 12)
    dpre = P.poison((M, N), "bf16")
    dbias = torch.empty(N, dtype=torch.float32, device="cuda")
    ws, nbytes = _workspace(fl, M, N, "bf16")
    fl.fl_drelu_bgrad(grad.cuda(), torch.from_numpy(mask.view(np.int32)).cuda(), dpre, dbias, M, N, "bf16", ws, nbytes)
    torch.cuda.synchronize()
    dv, db = oracle.drelu_bgrad(P.to64(grad), mask, N, "bf16")
    assert np.array_equal(P.to64(dpre), dv)
    _check_dbias(P.to64(dbias), db, np.abs(dv).sum(axis=0), M, what="drelu_bgrad 4096")


@pytest.mark.parametrize("M,N,dtype", [(300, 520, "bf16"), (257, 77, "f16"), (64, 1000, "f32"), (2048, 4096, "bf16")])
def test_dgelu_bgrad(fl, M, N, dtype):
    g = torch.Generator().manual_seed(M * 3 + N)
    v = (torch.randn(M, N, generator=g, dtype=torch.float32) * 3).to(P.TD[dtype])
    grad = _grad(M, N, dtype, M + 5 * N)
    dpre = P.poison((M, N), dtype)
    dbias = torch.empty(N, dtype=torch.float32, device="cuda")
    ws, nbytes = _workspace(fl, M, N, dtype)
    fl.fl_dgelu_bgrad(grad.cuda(), v.cuda(), dpre, dbias, M, N, dtype, ws, nbytes)
    torch.cuda.synchronize()
    g64, v64 = P.to64(grad), P.to64(v)
    dv, db = oracle.dgelu_bgrad(g64, v64, dtype)
    err = np.abs(P.to64(dpre) - dv)
    tol = P.ULP_REL[dtype] * np.abs(dv) + ULP_MIN[dtype] + 2 * GELU_GRAD_ABS * np.abs(g64)
    assert np.all(err <= tol), f"dgelu dpre error {err.max():.3e}"
    exact = g64 * oracle.gelu_erf_grad(v64)
    _check_dbias(P.to64(dbias), db, np.abs(exact).sum(axis=0), M, np.abs(g64).sum(axis=0), f"dgelu_bgrad {M}x{N}")


@pytest.mark.parametrize("M,N,K,out_dtype", [(300, 520, 200, "bf16"), (300, 520, 200, "f32"), (77, 1000, 1000, "bf16"),
                                             (257, 136, 768, "f16")])
def test_gelu_aux_forward_then_backward(fl, M, N, K, out_dtype):
    """GELU_AUX_BIAS stores v; the GELU backward takes it as its input."""
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 31, bias_dtype="bf16")
    ldo = -(-N // 8) * 8
    out = P.poison((M, ldo), out_dtype)
    vaux = P.poison((M, ldo), out_dtype)
    plan = fl.Plan(M, N, K, kind="GELU_AUX_BIAS", out_dtype=out_dtype, lda=inp["A"].shape[1],
                   ldb=inp["W"].shape[1], ldo=ldo)
    try:
        plan.execute(inp["A"].cuda(), inp["W"].cuda(), inp["bias"].cuda(), vaux, None, out)
        assert plan.check() == fl.FL_OK, fl.fl_last_error()
        info = plan.info()
    finally:
        plan.free()
    y, aux, v, absdot = P.oracle_linear(A=inp["A"], W=inp["W"], bias=inp["bias"], epilogue="GELU_AUX_BIAS",
                                        out_dtype=out_dtype, M=M, N=N, K=K)
    P.check_close(P.to64(out[:, :N]), y, out_dtype, absdot, f"GELU_AUX out {info}")
    P.check_close(P.to64(vaux[:, :N]), aux, out_dtype, absdot, f"GELU_AUX v {info}")
    assert torch.isnan(vaux[:, N:].float()).all(), "pre-activation written into the row padding"
    # backward from the stored v
    grad = _grad(M, N, out_dtype, 41, ld=ldo).cuda()
    dpre = P.poison((M, ldo), out_dtype)
    dbias = torch.empty(N, dtype=torch.float32, device="cuda")
    ws, nbytes = _workspace(fl, M, N, out_dtype)
    fl.fl_dgelu_bgrad(grad, vaux, dpre, dbias, M, N, out_dtype, ws, nbytes, ld_grad=ldo, ld_v=ldo, ld_dpre=ldo)
    torch.cuda.synchronize()
    g64, v64 = P.to64(grad[:, :N]), P.to64(vaux[:, :N])
    dv, db = oracle.dgelu_bgrad(g64, v64, out_dtype)
    err = np.abs(P.to64(dpre[:, :N]) - dv)
    assert np.all(err <= P.ULP_REL[out_dtype] * np.abs(dv) + ULP_MIN[out_dtype] + 2 * GELU_GRAD_ABS * np.abs(g64))
    exact = g64 * oracle.gelu_erf_grad(v64)
    _check_dbias(P.to64(dbias), db, np.abs(exact).sum(axis=0), M, np.abs(g64).sum(axis=0), "dgelu after GELU_AUX")


# ---------------------------------------------------------------- LayerNorm after the tail
def _ln_check(got, x64, g64, b64, eps, out_dtype, what):
    ref = oracle.layer_norm(x64, g64, b64, eps, out_dtype)
    mu = x64.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(((x64 - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    # fp32 mean and variance: |Δμ| ≲ 2^-20·max|x| of the row, |Δrstd|/rstd ≲ 2^-20
    tol = (2.0 ** -20) * np.abs(g64) * rstd * (np.abs(x64).max(axis=1, keepdims=True) + np.abs(x64 - mu)) \
        + 2 * P.ULP_REL[out_dtype] * np.abs(ref) + ULP_MIN[out_dtype]
    err = np.abs(got - ref)
    assert np.all(err <= tol), f"{what}: LayerNorm error {err.max():.3e} (bound there {tol.flat[err.argmax()]:.3e})"


@pytest.mark.parametrize("M,N,x_dtype,z_dtype,p_dtype,eps", [
    (300, 520, "f32", "f32", "f32", 1e-12), (64, 4096, "f32", "bf16", "bf16", 1e-5), (7, 77, "bf16", "bf16", "f32", 1e-5),
    (33, 20000, "f32", "f32", "f32", 1e-12), (2048, 4096, "f32", "bf16", "f32", 1e-12), (5, 1000, "f16", "f16", "f16", 1e-5),
    (16, 6000, "bf16", "f32", "bf16", 1e-5), (9, 5000, "f32", "f16", "f32", 1e-5), (3, 4097, "f32", "f32", "f32", 1e-5),
    # more rows than one resident wave: CTAs loop over rows (prefetching the next when aligned)
    (3000, 1032, "bf16", "f16", "f32", 1e-5), (4000, 300, "bf16", "bf16", "bf16", 1e-5),
    (1200, 4100, "f32", "f32", "f32", 1e-5), (2000, 6000, "bf16", "bf16", "f32", 1e-5),
    # whole vectors in warp 0 alone (the statistics merge warps without elements)
    (256, 40, "f32", "f32", "f32", 1e-5)])
def test_layernorm(fl, M, N, x_dtype, z_dtype, p_dtype, eps):
    g = torch.Generator().manual_seed(M + N)
    x = (torch.randn(M, N, generator=g) * 2 + 0.7).to(P.TD[x_dtype])
    gamma = (torch.rand(N, generator=g) + 0.5).to(P.TD[p_dtype])
    beta = torch.randn(N, generator=g).to(P.TD[p_dtype])
    z = P.poison((M, N), z_dtype)
    fl.fl_layernorm(x.cuda(), gamma.cuda(), beta.cuda(), z, M, N, x_dtype, z_dtype, p_dtype, eps=eps)
    torch.cuda.synchronize()
    _ln_check(P.to64(z), P.to64(x), P.to64(gamma)[None, :], P.to64(beta)[None, :], eps, z_dtype,
              f"LN {M}x{N} {x_dtype}->{z_dtype}")


@pytest.mark.parametrize("M,N", [(600, 4096), (300, 1000)])
def test_layernorm_large_offset(fl, M, N):
    # |μ|/σ ≈ 6000 per row: the per-warp two-pass sums and their merge keep the variance
    g = torch.Generator().manual_seed(N)
    x = torch.randn(M, N, generator=g, dtype=torch.float64) * 0.05 + 300.0
    x += torch.linspace(-20.0, 20.0, M, dtype=torch.float64)[:, None]
    x = x.float()
    gamma = (torch.rand(N, generator=g) + 0.5).float()
    beta = torch.randn(N, generator=g).float()
    z = P.poison((M, N), "bf16")
    fl.fl_layernorm(x.cuda(), gamma.cuda(), beta.cuda(), z, M, N, "f32", "bf16", "f32", eps=1e-5)
    torch.cuda.synchronize()
    _ln_check(P.to64(z), P.to64(x), P.to64(gamma)[None, :], P.to64(beta)[None, :], 1e-5, "bf16",
              f"LN {M}x{N} offset 300")


def test_layernorm_in_place_without_affine(fl):
    M, N = 100, 3000
    g = torch.Generator().manual_seed(9)
    x = torch.randn(M, N, generator=g) * 5
    buf = x.cuda()
    fl.fl_layernorm(buf, None, None, buf, M, N, "f32", "f32")
    torch.cuda.synchronize()
    _ln_check(P.to64(buf), P.to64(x), np.ones((1, N)), np.zeros((1, N)), 1e-12, "f32", "LN in place")


@pytest.mark.parametrize("ldx_pad,ldz_pad,param_off", [(0, 0, 1), (3, 0, 0), (0, 5, 0), (4, 4, 4)])
def test_layernorm_pitches_and_parameter_alignment(fl, ldx_pad, ldz_pad, param_off):
    """Row pitches and parameter offsets that switch between the vector and the element paths."""
    M, N = 37, 1032
    g = torch.Generator().manual_seed(ldx_pad * 100 + ldz_pad * 10 + param_off)
    x = torch.randn(M, N + ldx_pad, generator=g) * 3 - 1
    gfull = torch.rand(N + param_off, generator=g) + 0.5
    bfull = torch.randn(N + param_off, generator=g)
    gamma, beta = gfull.cuda()[param_off:], bfull.cuda()[param_off:]
    z = P.poison((M, N + ldz_pad), "bf16")
    fl.fl_layernorm(x.cuda(), gamma, beta, z, M, N, "f32", "bf16", "f32", eps=1e-5, ld_x=N + ldx_pad, ld_z=N + ldz_pad)
    torch.cuda.synchronize()
    _ln_check(P.to64(z)[:, :N], P.to64(x)[:, :N], P.to64(gfull[param_off:])[None, :],
              P.to64(bfull[param_off:])[None, :], 1e-5, "bf16", f"LN pitches {ldx_pad},{ldz_pad},{param_off}")
    if ldz_pad:
        assert torch.isnan(z[:, N:]).all(), "LN wrote the pitch pad"


def test_bert_tail_then_layernorm(fl):
    """bias -> GELU -> + residual -> x 0.5 in the fused layer, then LayerNorm of the rows."""
    w = workloads.get("tail_m512")
    inp = workloads.make_inputs(w, 0)
    out = torch.empty(w.M, w.N, dtype=torch.float32, device="cuda")
    plan = fl.Plan(w.M, w.N, w.K, kind=w.epilogue, out_dtype="f32", bias_dtype=w.bias_dtype, residual_dtype=w.dtype,
                   has_residual=True, scale=w.scale)
    try:
        plan.execute(inp["A"].cuda(), inp["W"].cuda(), inp["bias"].cuda(), None, inp["residual"].cuda(), out)
        assert plan.check() == fl.FL_OK, fl.fl_last_error()
    finally:
        plan.free()
    gamma = torch.ones(w.N, dtype=torch.float32, device="cuda")
    beta = torch.zeros(w.N, dtype=torch.float32, device="cuda")
    z = P.poison((w.M, w.N), "bf16")
    fl.fl_layernorm(out, gamma, beta, z, w.M, w.N, "f32", "bf16", "f32", eps=1e-12)
    torch.cuda.synchronize()
    sel = P.sample_rows(w.M, 64, 2)
    y, _, _, absdot = P.oracle_linear(A=inp["A"], W=inp["W"], bias=inp["bias"], residual=inp["residual"],
                                      scale=w.scale, epilogue=w.epilogue, out_dtype="f32", M=w.M, N=w.N, K=w.K,
                                      rows=sel)
    # the layer output against the oracle, then LayerNorm of the GPU's own rows
    P.check_close(P.to64(out)[sel], y, "f32", absdot, "tail_m512 layer")
    _ln_check(P.to64(z)[sel], P.to64(out)[sel], np.ones((1, w.N)), np.zeros((1, w.N)), 1e-12, "bf16",
              "tail_m512 LayerNorm")


def test_bounded_wait_failure_path(fl):
    """A wait that nothing satisfies gives up after its limit and reports FL_ERR_TIMEOUT;
    the context stays usable (a layer runs and matches the oracle right after)."""
    import time
    t0 = time.perf_counter()
    assert fl.fl_wait_selftest(20_000_000) == fl.FL_ERR_TIMEOUT, fl.fl_last_error()
    assert time.perf_counter() - t0 < 5.0
    got = P.run_linear(fl, M=130, N=200, K=64, dtype="bf16", epilogue="RELU_BIAS", out_dtype="bf16",
                       **_small_layer_inputs())
    y, _, _, absdot = P.oracle_linear(epilogue="RELU_BIAS", out_dtype="bf16", M=130, N=200, K=64,
                                      **{k: v for k, v in _small_layer_inputs().items() if k in ("A", "W", "bias")})
    P.check_close(got["out"], y, "bf16", absdot, "layer after the self-test")


def _small_layer_inputs():
    inp = workloads.ragged_linear_inputs(130, 200, 64, "bf16", 77, bias_dtype="bf16")
    return {"A": inp["A"], "W": inp["W"], "bias": inp["bias"]}
