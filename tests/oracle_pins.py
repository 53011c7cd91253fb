"""Pins that tie the oracle to something other than itself.

Each ``pin_*`` takes an oracle namespace ``o`` (the real ``oracle`` package,
or a deliberately broken copy in the mutation tests) and raises
AssertionError when the oracle disagrees with:
  * brute force on tiny inputs (pure-Python loops),
  * closed forms / series from the mathematics (Maclaurin series of erf),
  * identities (GELU(x) − GELU(−x) = x, relu(v) − relu(−v) = v, ...),
  * constants printed on the pages (tests/golden/page_constants.json),
  * an independent library routine for a special case (torch fp64 F.linear,
    F.gelu, dtype casts).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_constants.json")


def _golden():
    with open(GOLDEN, encoding="utf-8") as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- GEMM
def pin_gemm_hand_example(o):
    # [[1,2,3],[4,5,6]] · [[1,0,1],[0,1,1]]ᵀ = [[4,5],[10,11]]
    A = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]])
    W = np.array([[1.0, 0.0, 1.0], [0.0, 1.0, 1.0]])
    acc = o.gemm(A, W)
    assert np.array_equal(acc, np.array([[4.0, 5.0], [10.0, 11.0]])), acc
    # Same product with the second operand stored [K,N].
    acc2 = o.gemm(A, W.T.copy(), b_major=1)
    assert np.array_equal(acc2, acc), acc2


def pin_gemm_brute_force(o):
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (17, 33, 65), (2, 9, 4)]:
        r = _rng(M * 1000 + N * 10 + K)
        A = r.standard_normal((M, K))
        W = r.standard_normal((N, K))
        ref = np.zeros((M, N))
        for m in range(M):
            for n in range(N):
                s = 0.0
                for k in range(K):
                    s += A[m, k] * W[n, k]
                ref[m, n] = s
        got = o.gemm(A, W)
        assert got.shape == (M, N)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), (M, N, K)
        gotb = o.gemm(A, W.T.copy(), b_major=1)
        assert np.allclose(gotb, ref, rtol=1e-12, atol=1e-12), (M, N, K, "b_major")


# ---------------------------------------------------------------- bias
def pin_bias_broadcast_axes(o):
    g = _golden()["epilog_example"]
    Mo, Ki = g["W"]
    _, Nb = g["x"]
    r = _rng(1)
    bias_m = r.standard_normal(Mo)
    # With A = 0 the result is the bias broadcast over every column (axis M).
    v = o.add_bias(o.gemm(np.zeros((Mo, Ki)), r.standard_normal((Ki, Nb)), b_major=1), bias_m, axis=1)
    assert v.shape == tuple(g["result"])
    assert np.array_equal(v, np.repeat(bias_m[:, None], Nb, axis=1))
    # Linear form x·Wᵀ: bias per output feature n, broadcast over rows.
    bias_n = r.standard_normal(7)
    v2 = o.add_bias(np.zeros((5, 7)), bias_n, axis=0)
    assert np.array_equal(v2, np.repeat(bias_n[None, :], 5, axis=0))


def pin_linear_vs_torch(o):
    g = _golden()["linear_gelu_unit_test"]
    M, K = 64, g["x"][1]            # a row slice of the page's unit-test shape
    N = 96
    gen = torch.Generator().manual_seed(3)
    x = torch.randn(M, K, generator=gen, dtype=torch.float64)
    w = torch.randn(N, K, generator=gen, dtype=torch.float64)
    b = torch.randn(N, generator=gen, dtype=torch.float64)
    ref_lin = F.linear(x, w, b).numpy()
    v = o.add_bias(o.gemm(x.numpy(), w.numpy()), b.numpy(), axis=0)
    assert np.allclose(v, ref_lin, rtol=1e-12, atol=1e-10)
    ref_gelu = F.gelu(F.linear(x, w, b)).numpy()
    assert np.allclose(o.gelu_erf(v), ref_gelu, rtol=1e-12, atol=1e-12)
    ref_tanh = F.gelu(F.linear(x, w, b), approximate="tanh").numpy()
    assert np.allclose(o.gelu_tanh(v), ref_tanh, rtol=1e-12, atol=1e-12)
    assert np.array_equal(o.relu(ref_lin), F.relu(torch.from_numpy(ref_lin)).numpy())


# ---------------------------------------------------------------- activations
def pin_relu_identities(o):
    v = np.linspace(-5, 5, 1001)
    r = o.relu(v)
    assert np.array_equal(r - o.relu(-v), v)           # relu(v) − relu(−v) = v
    assert np.array_equal(o.relu(r), r)                # idempotent
    assert np.all(r >= 0) and o.relu(np.array([0.0]))[0] == 0.0


def _erf_series(x: float) -> float:
    """Maclaurin series erf(x) = 2/√π Σ (−1)^n x^(2n+1) / (n!(2n+1)), |x| ≤ 3."""
    s, term, n = 0.0, x, 0
    while True:
        add = term / (2 * n + 1)
        s += add
        if abs(add) < 1e-18 * max(1.0, abs(s)):
            break
        n += 1
        term *= -x * x / n
    return 2.0 / math.sqrt(math.pi) * s


def pin_gelu_erf_series(o):
    xs = np.array([-3.0, -2.0, -1.0, -0.5, -0.1, 0.0, 0.1, 0.5, 1.0, 1.5, 2.0, 3.0])
    ref = np.array([0.5 * x * (1.0 + _erf_series(x / math.sqrt(2.0))) for x in xs])
    got = o.gelu_erf(xs)
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-15), np.max(np.abs(got - ref))
    assert got[xs == 0.0][0] == 0.0


def pin_gelu_closed_forms(o):
    """GELU(x) = x·Φ(x) at points where Φ is tabulated: the standard normal CDF to 15 digits
    (Abramowitz & Stegun, Table 26.1): Φ(0.5) = 0.691462461274013, Φ(1) = 0.841344746068543,
    Φ(2) = 0.977249868051821, and Φ(−x) = 1 − Φ(x)."""
    table = {0.5: 0.691462461274013, 1.0: 0.841344746068543, 2.0: 0.977249868051821}
    for x, phi in table.items():
        got = o.gelu_erf(np.array([x, -x]))
        assert abs(got[0] - x * phi) < 1e-14, (x, got[0])
        assert abs(got[1] - (-x) * (1.0 - phi)) < 1e-14, (-x, got[1])


def pin_gelu_identities(o):
    x = np.linspace(-8, 8, 4001)
    for f in (o.gelu_erf, o.gelu_tanh):
        d = f(x) - f(-x)
        assert np.allclose(d, x, rtol=0, atol=1e-12)     # odd part is x/2 on each side
        big = np.array([30.0, 40.0])
        assert np.allclose(f(big), big) and np.allclose(f(-big), 0.0, atol=1e-30)
    # dGELU/dx at 0 is 1/2 for both forms
    h = 1e-6
    for f in (o.gelu_erf, o.gelu_tanh):
        slope = (f(np.array([h]))[0] - f(np.array([-h]))[0]) / (2 * h)
        assert abs(slope - 0.5) < 1e-9


def pin_gelu_tanh_page_constants(o):
    g = _golden()
    c, a = g["gelu_tanh_c"]["value"], g["gelu_tanh_a"]["value"]
    x = np.linspace(-6, 6, 2401)
    # 0.5(1 + tanh(u)) = 1 / (1 + exp(−2u)): an algebraically different route
    # with the constants the pages print.
    u = c * (x + a * x ** 3)
    ref = x / (1.0 + np.exp(-2.0 * u))
    got = o.gelu_tanh(x)
    # 0.79788456 is √(2/π) rounded to 8 digits: allow the difference it makes.
    assert np.allclose(got, ref, rtol=0, atol=5e-8), np.max(np.abs(got - ref))
    bound = g["gelu_approx_error_bound"]["value"]
    xx = np.linspace(-10, 10, 20001)
    err = np.max(np.abs(o.gelu_tanh(xx) - o.gelu_erf(xx)))
    assert err < bound, err
    assert err > 1e-4, err      # the two forms are genuinely different functions


# ---------------------------------------------------------------- aux mask
def pin_aux_mask_layout(o):
    v = np.full((2, 40), -1.0)
    v[0, [0, 5, 33]] = 2.0
    v[1, 31] = 0.5
    v[1, 39] = 1e-300
    v[1, 7] = 0.0             # ReLU'(0) = 0: not set
    m = o.relu_aux_mask(v)
    assert m.dtype == np.uint32 and m.shape == (2, 2)
    assert m[0, 0] == (1 | (1 << 5)) and m[0, 1] == (1 << 1)
    assert m[1, 0] == (1 << 31) and m[1, 1] == (1 << 7)


def pin_aux_mask_popcount(o):
    r = _rng(5)
    v = r.standard_normal((9, 77))
    m = o.relu_aux_mask(v)
    pop = np.array([sum(bin(int(w)).count("1") for w in row) for row in m])
    assert np.array_equal(pop, (v > 0).sum(axis=1))
    # padding bits of the last word are zero: columns 77..95 do not exist
    assert np.all((m[:, 2].astype(np.uint64) >> np.uint64(77 - 64)) == 0)


# ---------------------------------------------------------------- tail, dReLU, GeGLU
def pin_residual_scale(o):
    r = _rng(6)
    M, N, K = 4, 6, 5
    res = o.round_to(r.standard_normal((M, N)), "bf16")
    y, _, _ = o.fused_linear(np.zeros((M, K)), np.zeros((N, K)), np.zeros(N), epilogue="GELU_BIAS",
                             out_dtype="f32", residual=res, scale=0.5)
    assert np.array_equal(y, 0.5 * res)          # gelu(0)=0, so y = 0.5·r exactly
    # order: (gelu(v) + r)·0.5, not gelu(v)+0.5r nor gelu(v+r)
    A = np.eye(3)
    W = np.eye(3)
    b = np.zeros(3)
    resid = np.array([[1.0, 1.0, 1.0]] * 3)
    y2, _, _ = o.fused_linear(A, W, b, epilogue="GELU_BIAS", out_dtype="f32", residual=resid, scale=0.5)
    g1 = 0.5 * (1.0 + _erf_series(1.0 / math.sqrt(2.0)))
    assert abs(y2[0, 0] - np.float32(0.5 * (g1 + 1.0))) < 1e-7
    assert abs(y2[0, 1] - 0.5) < 1e-7


def pin_drelu(o):
    r = _rng(7)
    M, N = 5, 70
    v = r.standard_normal((M, N))
    grad = o.round_to(r.standard_normal((M, N)), "bf16")
    d = o.drelu(grad, o.relu_aux_mask(v), N, "bf16")
    assert np.array_equal(d, np.where(v > 0, grad, 0.0))


def pin_geglu_identity(o):
    r = _rng(8)
    M, K = 6, 16
    x = o.round_to(r.standard_normal((M, K)), "bf16")
    Wg = o.round_to(r.standard_normal((K, K)) * 0.3, "bf16")
    h = o.geglu_h(x, Wg, np.eye(K), "f32")         # Wu = I  ⇒  u = x
    g = np.zeros((M, K))
    for m in range(M):
        for n in range(K):
            g[m, n] = sum(x[m, k] * Wg[n, k] for k in range(K))
    ref = F.gelu(torch.from_numpy(g), approximate="tanh").numpy() * x
    assert np.allclose(h, o.round_to(ref, "f32"), rtol=1e-6, atol=1e-7)
    hh, y = o.geglu_mlp(x, Wg, np.eye(K), np.eye(K), "f32")   # Wd = I  ⇒  y = h
    assert np.array_equal(y, hh)


def _geglu_mlp_loops(x, Wg, Wu, Wd, round_h, round_fn):
    """GeGLU MLP by per-element loops: h = gelu_tanh(x·Wgᵀ)·(x·Wuᵀ) with math.tanh, optionally
    rounded to bf16, then y[m,j] = Σ_n h[m,n]·Wd[j,n] (Wd is the down projection's [K, N] weight)."""
    M, K = x.shape
    N, J = Wg.shape[0], Wd.shape[0]
    c = math.sqrt(2.0 / math.pi)
    h = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            g = sum(x[m, k] * Wg[n, k] for k in range(K))
            u = sum(x[m, k] * Wu[n, k] for k in range(K))
            h[m, n] = 0.5 * g * (1.0 + math.tanh(c * (g + 0.044715 * g ** 3))) * u
    if round_h:
        h = round_fn(h)
    y = np.zeros((M, J))
    for m in range(M):
        for j in range(J):
            y[m, j] = sum(h[m, n] * Wd[j, n] for n in range(N))
    return round_fn(h), round_fn(y)


def pin_geglu_mlp_bf16_brute_force(o):
    """The whole MLP in bf16 against loops, with a rectangular (K≠N) and a square non-symmetric
    down-projection weight: h is rounded to bf16 before the down projection (h is a bf16 tensor),
    and Wd is read as [out, in].  The inputs are chosen so that skipping the rounding of h
    changes y (checked here, so the pin stays sensitive to it)."""
    def bf16(v):
        # torch's float32 -> bfloat16 cast on values first rounded to float32 (ties are
        # not reached by these sums of products of bf16 values at this size)
        return torch.from_numpy(np.asarray(v, np.float64)).to(torch.float32).to(torch.bfloat16) \
            .to(torch.float64).numpy()
    for (M, K, N, seed) in [(4, 6, 10, 100), (3, 7, 7, 105)]:
        r = _rng(seed)
        x = bf16(r.standard_normal((M, K)))
        Wg = bf16(r.standard_normal((N, K)) * 0.5)
        Wu = bf16(r.standard_normal((N, K)) * 0.5)
        Wd = bf16(r.standard_normal((K, N)) * 0.5)
        h_ref, y_ref = _geglu_mlp_loops(x, Wg, Wu, Wd, True, bf16)
        _, y_unrounded_h = _geglu_mlp_loops(x, Wg, Wu, Wd, False, bf16)
        assert (y_ref != y_unrounded_h).any()      # the case distinguishes the two readings
        if K == N:
            assert not np.array_equal(Wd, Wd.T)    # a transposed Wd gives other values
        h, y = o.geglu_mlp(x, Wg, Wu, Wd, "bf16")
        assert np.array_equal(h, h_ref), (M, K, N)
        assert np.array_equal(y, y_ref), (M, K, N)


def pin_gelu_sigmoid_page_form(o):
    """x·σ(1.702x) with the page's constant, per element against math.exp."""
    k = _golden()["gelu_sigmoid_k"]["value"]
    v = np.linspace(-20.0, 20.0, 161)
    y = o.gelu_sigmoid(v)
    for x, got in zip(v, y):
        assert abs(got - x / (1.0 + math.exp(-k * x))) <= 1e-15 * max(1.0, abs(x))


def pin_gelu_sigmoid_identities(o):
    v = np.linspace(-8.0, 8.0, 161)
    # σ(z) + σ(-z) = 1  ⇒  f(v) − f(−v) = v
    assert np.max(np.abs(o.gelu_sigmoid(v) - o.gelu_sigmoid(-v) - v)) < 1e-14
    assert o.gelu_sigmoid(np.array([0.0]))[0] == 0.0
    assert abs(o.gelu_sigmoid(np.array([60.0]))[0] - 60.0) < 1e-12
    assert abs(o.gelu_sigmoid(np.array([-60.0]))[0]) < 1e-40
    # the activation kind routes to it
    assert np.array_equal(o.activation(v, "GELU_SIGMOID_BIAS"), o.gelu_sigmoid(v))


def pin_layer_norm(o):
    r = _rng(15)
    M, N = 6, 40
    x = r.standard_normal((M, N)) * 3 + 1.5
    g = r.standard_normal(N)
    b = r.standard_normal(N)
    z = o.layer_norm(x, g, b, 1e-5, "f32")
    # per row against loops
    for m in range(M):
        mu = sum(x[m]) / N
        var = sum((v - mu) ** 2 for v in x[m]) / N
        for n in range(N):
            ref = (x[m, n] - mu) / math.sqrt(var + 1e-5) * g[n] + b[n]
            assert abs(z[m, n] - np.float32(ref)) <= 1e-6 * max(1.0, abs(ref))
    # γ = 1, β = 0: each row has mean 0 and population variance var/(var + ε)
    z1 = o.layer_norm(x, np.ones(N), np.zeros(N), 0.0, "f32")
    assert np.max(np.abs(z1.mean(axis=1))) < 1e-6
    assert np.max(np.abs(z1.var(axis=1) - 1.0)) < 1e-5
    # against torch's layer_norm in fp64
    zt = F.layer_norm(torch.from_numpy(x), (N,), torch.from_numpy(g), torch.from_numpy(b), eps=1e-12).numpy()
    assert np.max(np.abs(o.layer_norm(x, g, b, 1e-12, "f32") - o.round_to(zt, "f32"))) < 1e-6
    # invariant to shifting the row
    assert np.max(np.abs(o.layer_norm(x + 100.0, g, b, 1e-5, "f32") - z)) < 1e-5


def pin_bias_grad_brute_force(o):
    r = _rng(11)
    M, N = 7, 9
    dv = r.standard_normal((M, N))
    db = o.bias_grad(dv)
    for n in range(N):
        assert abs(db[n] - sum(dv[m, n] for m in range(M))) < 1e-12
    assert np.array_equal(o.bias_grad(np.ones((5, 3))), np.full(3, 5.0))


def pin_drelu_bgrad(o):
    r = _rng(12)
    M, N = 6, 45
    v = r.standard_normal((M, N))
    grad = o.round_to(r.standard_normal((M, N)), "bf16")
    dv, db = o.drelu_bgrad(grad, o.relu_aux_mask(v), N, "bf16")
    for n in range(N):
        want = sum(grad[m, n] for m in range(M) if v[m, n] > 0)
        assert abs(db[n] - want) < 1e-12, n
    assert np.array_equal(dv, np.where(v > 0, grad, 0.0))


def pin_gelu_grad_finite_difference(o):
    """GELU' against a central difference of GELU (fp64, h = 1e-5: error ~1e-10)."""
    v = np.linspace(-9.0, 9.0, 721)
    h = 1e-5
    fd = (o.gelu_erf(v + h) - o.gelu_erf(v - h)) / (2 * h)
    assert np.max(np.abs(o.gelu_erf_grad(v) - fd)) < 1e-8


def pin_gelu_grad_identities(o):
    v = np.linspace(-6.0, 6.0, 241)
    # Φ(v) + Φ(-v) = 1 and the v·φ(v) terms cancel: GELU'(v) + GELU'(-v) = 1
    assert np.max(np.abs(o.gelu_erf_grad(v) + o.gelu_erf_grad(-v) - 1.0)) < 1e-14
    assert o.gelu_erf_grad(np.array([0.0]))[0] == 0.5
    assert abs(o.gelu_erf_grad(np.array([40.0]))[0] - 1.0) < 1e-15
    assert abs(o.gelu_erf_grad(np.array([-40.0]))[0]) < 1e-15
    # GELU' exceeds 1 just above zero (the maximum is near v = 1.4)
    assert o.gelu_erf_grad(np.array([1.4]))[0] > 1.12


def pin_dgelu_bgrad(o):
    r = _rng(13)
    M, N = 5, 33
    v = o.round_to(r.standard_normal((M, N)) * 2, "bf16")
    grad = o.round_to(r.standard_normal((M, N)), "bf16")
    dv, db = o.dgelu_bgrad(grad, v, "bf16")
    assert np.array_equal(dv, o.dgelu(grad, v, "bf16"))
    for m in range(M):
        for n in range(N):
            x = v[m, n]
            g = 0.5 * (1 + math.erf(x / math.sqrt(2.0))) + x * math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
            assert dv[m, n] == o.round_to(np.array([grad[m, n] * g]), "bf16")[0]
    for n in range(N):
        x = v[:, n]
        want = sum(grad[m, n] * (0.5 * (1 + math.erf(x[m] / math.sqrt(2.0)))
                                 + x[m] * math.exp(-x[m] ** 2 / 2) / math.sqrt(2 * math.pi)) for m in range(M))
        assert abs(db[n] - want) < 1e-12


def pin_gelu_aux_stores_preactivation(o):
    r = _rng(14)
    M, N, K = 4, 19, 6
    A = r.standard_normal((M, K))
    W = r.standard_normal((N, K))
    b = r.standard_normal(N)
    y, aux, v = o.fused_linear(A, W, b, epilogue="GELU_AUX_BIAS", out_dtype="bf16")
    for m in range(M):
        for n in range(N):
            acc = sum(A[m, k] * W[n, k] for k in range(K)) + b[n]
            assert aux[m, n] == o.round_to(np.array([acc]), "bf16")[0]
            assert y[m, n] == o.round_to(np.array([0.5 * acc * (1 + math.erf(acc / math.sqrt(2.0)))]), "bf16")[0]


# ---------------------------------------------------------------- rounding
def pin_round_to(o):
    one = 1.0
    # bf16 ties: 1+2^-8 lies halfway between 1 and 1+2^-7 -> even (1.0);
    # 1+3·2^-8 lies halfway between 1+2^-7 and 1+2^-6 -> even (1+2^-6).
    t = np.array([one + 2 ** -8, one + 3 * 2 ** -8, -(one + 2 ** -8), 0.0, -0.0])
    assert np.array_equal(o.round_to(t, "bf16"), np.array([1.0, 1.0 + 2 ** -6, -1.0, 0.0, -0.0]))
    t16 = np.array([one + 2 ** -11, one + 3 * 2 ** -11, 65519.0, 65520.0, 2.0 ** -25, 3 * 2.0 ** -26])
    exp16 = np.array([1.0, 1.0 + 2 ** -9, 65504.0, np.inf, 0.0, 2.0 ** -24])
    assert np.array_equal(o.round_to(t16, "f16"), exp16), o.round_to(t16, "f16")
    # against torch's casts on random non-tie values across many binades
    r = _rng(9)
    x = r.standard_normal(20000) * np.exp2(r.integers(-30, 30, 20000))
    tb = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    x32 = x.astype(np.float32).astype(np.float64)     # exact fp32 values: no double rounding
    assert np.array_equal(o.round_to(x32, "bf16"), tb)
    xs = x32 * 1e-4
    th = torch.from_numpy(xs).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(o.round_to(xs, "f16"), th)
    assert np.array_equal(o.round_to(x, "f32"), x32)


def pin_fused_brute_force(o):
    """Every epilogue on a tiny case against per-element loops (math.erf / math.tanh)."""
    r = _rng(10)
    M, N, K = 3, 37, 5
    A = r.standard_normal((M, K))
    W = r.standard_normal((N, K))
    b = r.standard_normal(N)
    res = r.standard_normal((M, N))
    c = math.sqrt(2.0 / math.pi)
    acts = {
        "NONE": lambda v: v, "BIAS": lambda v: v, "RELU_BIAS": lambda v: max(v, 0.0),
        "RELU_AUX_BIAS": lambda v: max(v, 0.0),
        "GELU_BIAS": lambda v: 0.5 * v * (1 + math.erf(v / math.sqrt(2.0))),
        "GELU_TANH_BIAS": lambda v: 0.5 * v * (1 + math.tanh(c * (v + 0.044715 * v ** 3))),
        "GELU_SIGMOID_BIAS": lambda v: v / (1.0 + math.exp(-1.702 * v)),
    }
    for epi, f in acts.items():
        y, aux, v = o.fused_linear(A, W, b, epilogue=epi, out_dtype="f32", residual=res, scale=0.25)
        for m in range(M):
            for n in range(N):
                acc = sum(A[m, k] * W[n, k] for k in range(K)) + (0.0 if epi == "NONE" else b[n])
                ref = np.float32((f(acc) + res[m, n]) * 0.25)
                assert abs(y[m, n] - ref) <= 1e-6 * max(1.0, abs(ref)), (epi, m, n)
                if epi == "RELU_AUX_BIAS":
                    bit = (int(aux[m, n // 32]) >> (n % 32)) & 1
                    assert bit == (1 if acc > 0 else 0)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
