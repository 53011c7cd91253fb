"""fp64 CPU oracle of y = act(A·Wᵀ + bias) and its relatives — TEST INFRASTRUCTURE.

Each function states the passage it follows (page keys are defined in
``oracle/__init__.py``).  Arrays are numpy; inputs are the values actually
stored on the device (already rounded to fp16/bf16/fp32), widened exactly to
float64.  All arithmetic is float64; a result is rounded exactly once, at the
end, to the output dtype (round-to-nearest-even), which is the plain
definition the fused kernel reaches up to summation order.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

# [gelu] §2.2.2 writes the constant as math.sqrt(2/math.pi); [mhc] §4.2 prints
# it to eight digits as 0.79788456.  The oracle uses the exact value.
GELU_TANH_C = math.sqrt(2.0 / math.pi)
# [gelu] §2.2.2 and [mhc] §4.2: the cubic coefficient of the tanh form.
GELU_TANH_A = 0.044715
# [gelu] §2.2.2, "approximation 1": the sigmoid slope of x·σ(1.702x).
GELU_SIGMOID_K = 1.702


def gemm(A: np.ndarray, W: np.ndarray, b_major: int = 0) -> np.ndarray:
    """acc[m,n] = Σ_k A[m,k]·W[n,k] in float64.

    [mlp] "nn.Linear 的底層真相": addmm(bias, x, weight) = x @ weight.T + bias,
    the transpose being a stride swap only.  With ``b_major=1`` the second
    operand is stored [K,N] (the [epilog] code example's W·x with x [784,256]),
    so acc = A @ B.  numpy's float64 matmul is the library primitive here.
    """
    A = np.asarray(A, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    if b_major:
        assert A.shape[1] == W.shape[0], (A.shape, W.shape)
        return A @ W
    assert A.shape[1] == W.shape[1], (A.shape, W.shape)
    return A @ W.T


def add_bias(acc: np.ndarray, bias: np.ndarray, axis: int = 0) -> np.ndarray:
    """v = acc + bias broadcast, in float64 before any rounding.

    [epilog] ¶ on epilog_inputs: the bias has the length of the result's
    output-feature dimension and is broadcast over the other one.  For the
    Linear form x·Wᵀ that is the column index n (``axis=0``: bias[n]); for the
    page's own W·x example the output features are the rows (``axis=1``:
    bias[m], shape (100,) broadcast over 256 columns).
    """
    b = np.asarray(bias, dtype=np.float64)
    if axis == 0:
        assert b.shape == (acc.shape[1],), (b.shape, acc.shape)
        return acc + b[None, :]
    assert b.shape == (acc.shape[0],), (b.shape, acc.shape)
    return acc + b[:, None]


def relu(v: np.ndarray) -> np.ndarray:
    """max(v, 0) — [epilog] RELU_BIAS code example, y = relu(Wx + B)."""
    return np.where(v > 0.0, v, 0.0)


def gelu_erf(v: np.ndarray) -> np.ndarray:
    """Exact GELU: x·Φ(x) = 0.5·x·(1 + erf(x/√2)) — [gelu] §1 and §2.1."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + _erf(v / math.sqrt(2.0)))


def gelu_tanh(v: np.ndarray) -> np.ndarray:
    """tanh form: 0.5·x·(1 + tanh(√(2/π)·(x + 0.044715·x³))) — [gelu] §2.2.2, [mhc] §4.2."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + np.tanh(GELU_TANH_C * (v + GELU_TANH_A * v * v * v)))


def gelu_sigmoid(v: np.ndarray) -> np.ndarray:
    """Sigmoid form: x·σ(1.702·x) = x / (1 + e^(-1.702·x)) — [gelu] §2.2.2, approximation 1."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-GELU_SIGMOID_K * v))


def activation(v: np.ndarray, kind: str) -> np.ndarray:
    """Apply the activation named by an epilogue kind (bias-only kinds are identity)."""
    if kind in ("NONE", "BIAS"):
        return v
    if kind in ("RELU_BIAS", "RELU_AUX_BIAS", "RELU"):
        return relu(v)
    if kind in ("GELU_BIAS", "GELU_AUX_BIAS", "GELU"):
        return gelu_erf(v)
    if kind in ("GELU_TANH_BIAS", "GELU_TANH"):
        return gelu_tanh(v)
    if kind in ("GELU_SIGMOID_BIAS", "GELU_SIGMOID"):
        return gelu_sigmoid(v)
    raise ValueError(kind)


def relu_aux_mask(v: np.ndarray) -> np.ndarray:
    """Bit-packed ReLU mask of the pre-activation v, [M, ceil(N/32)] uint32.

    [epilog] RELU_AUX_BIAS: the forward pass also emits the ReLU mask used by
    the backward pass.  The page does not fix a layout; the one used here is
    row-major words, bit j of word w of row m set iff v[m, 32w+j] > 0
    (least-significant bit first; ReLU'(0) = 0; padding bits zero).
    """
    M, N = v.shape
    W = (N + 31) // 32
    out = np.zeros((M, W), dtype=np.uint64)
    pos = v > 0.0
    for n in range(N):
        out[:, n // 32] |= pos[:, n].astype(np.uint64) << np.uint64(n % 32)
    return out.astype(np.uint32)


def residual_scale(a: np.ndarray, residual, scale: float) -> np.ndarray:
    """y = (a + residual)·scale — [mhc] §2.2's chain 'residual Add, multiply by a constant'.

    The order (add the residual after the activation, then scale) is the
    reading of the BERT-tail workload: bias → GELU → +residual → ×0.5.
    """
    y = a
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    if scale != 1.0:
        y = y * float(scale)
    return y


def _round_significand(x: np.ndarray, sig_bits: int, min_exp: int, max_finite: float) -> np.ndarray:
    """Round float64 values to a binary format with ``sig_bits`` significand bits (RNE).

    The quantum of x = f·2^e (f in [0.5,1)) is 2^(e - sig_bits), floored at the
    subnormal quantum 2^min_exp; np.rint rounds half to even.  Values whose
    rounded magnitude exceeds the format's largest finite value become ±inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0.0)
    _, e = np.frexp(x[fin])
    q = np.maximum(e - sig_bits, min_exp).astype(np.float64)
    r = np.rint(np.ldexp(x[fin], (-q).astype(np.int64))) * np.exp2(q)
    r = np.where(np.abs(r) > max_finite, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 x once to the storage dtype; returns float64 holding those values.

    bf16: 8 significand bits, subnormal quantum 2^-133, max 0x7F7F = 3.3895e38.
    f16: 11 significand bits, subnormal quantum 2^-24, max 65504.
    f32: numpy's own float64→float32 cast (IEEE RNE).
    """
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return _round_significand(x, 8, -133, float.fromhex("0x1.fep127"))
    if dtype == "f16":
        return _round_significand(x, 11, -24, 65504.0)
    raise ValueError(dtype)


def fused_linear(A, W, bias=None, *, epilogue: str, out_dtype: str, bias_axis: int = 0,
                 b_major: int = 0, residual=None, scale: float = 1.0):
    """One fused linear layer: returns (y_rounded, aux_mask_or_None, v).

    v = A·Wᵀ + bias (fp64, bias added before any rounding, as the [epilog] page
    describes the epilog acting on the FP32 result); a = act(v);
    y = round_out((a + residual)·scale); aux = relu_aux_mask(v) for RELU_AUX_BIAS,
    and for GELU_AUX_BIAS the pre-activation itself, rounded once to out_dtype
    (the stored input of the GELU backward, see ``dgelu``).
    """
    v = gemm(A, W, b_major)
    if bias is not None and epilogue != "NONE":
        v = add_bias(v, bias, bias_axis)
    a = activation(v, epilogue)
    y = residual_scale(a, residual, scale)
    aux = None
    if epilogue == "RELU_AUX_BIAS":
        aux = relu_aux_mask(v)
    elif epilogue == "GELU_AUX_BIAS":
        aux = round_to(v, out_dtype)
    return round_to(y, out_dtype), aux, v


def geglu_h(x, Wg, Wu, out_dtype: str = "bf16"):
    """h = gelu_tanh(x·Wgᵀ) · (x·Wuᵀ), rounded once to out_dtype.

    [mlp] "GeGLU MLP 的五個 GPU Kernel": gate_proj and up_proj, GeLU on the
    gate, elementwise product; Liger's kernel is the tanh form.
    """
    g = gemm(x, Wg)
    u = gemm(x, Wu)
    return round_to(gelu_tanh(g) * u, out_dtype)


def geglu_mlp(x, Wg, Wu, Wd, out_dtype: str = "bf16"):
    """(h, y): h as in ``geglu_h`` (a bf16 tensor), y = round(h·Wdᵀ) — [mlp] down_proj."""
    h = geglu_h(x, Wg, Wu, out_dtype)
    y = round_to(gemm(h, Wd), out_dtype)
    return h, y


def drelu(grad, aux: np.ndarray, N: int, out_dtype: str = "bf16"):
    """dpre[m,n] = grad[m,n] · bit(m,n) — the backward use of the [epilog] RELU_AUX_BIAS mask.

    Multiplying by 0 or 1 is exact, so the rounding is the identity for a
    grad already stored in out_dtype.
    """
    grad = np.asarray(grad, dtype=np.float64)
    M = grad.shape[0]
    bits = np.zeros((M, N), dtype=np.float64)
    for n in range(N):
        bits[:, n] = ((aux[:, n // 32].astype(np.uint64) >> np.uint64(n % 32)) & np.uint64(1)).astype(np.float64)
    return round_to(grad[:, :N] * bits, out_dtype)


# ---------------------------------------------------------------- backward of the fused layer
# [epilog]: the RELU_AUX_BIAS epilog keeps a ReLU mask in the forward pass so that the
# backward pass computes its gradient efficiently; [gelu] §2.2.1: when Linear+GELU is
# rewritten into one fused operator, the backward gradient must be fused as well.  For
# y = act(v), v = x·Wᵀ + b with b broadcast over the rows m, the chain rule gives
#   dv[m,n] = dy[m,n] · act'(v[m,n])   and   db[n] = Σ_m dv[m,n].


def bias_grad(dv: np.ndarray) -> np.ndarray:
    """db[n] = Σ_m dv[m,n] in float64 (the bias is added to every row m of v)."""
    return np.asarray(dv, dtype=np.float64).sum(axis=0)


def drelu_bgrad(grad, aux: np.ndarray, N: int, out_dtype: str = "bf16"):
    """(dv, db): dv = ``drelu`` (grad times the mask bit, exact) and db = Σ_m dv in float64."""
    dv = drelu(grad, aux, N, out_dtype)
    return dv, bias_grad(dv)


def gelu_erf_grad(v: np.ndarray) -> np.ndarray:
    """d/dv [v·Φ(v)] = Φ(v) + v·φ(v), φ(v) = e^(-v²/2)/√(2π) — the derivative of [gelu] §1's GELU."""
    v = np.asarray(v, dtype=np.float64)
    Phi = 0.5 * (1.0 + _erf(v / math.sqrt(2.0)))
    phi = np.exp(-0.5 * v * v) / math.sqrt(2.0 * math.pi)
    return Phi + v * phi


def dgelu(grad, v, out_dtype: str = "bf16"):
    """dv = grad · GELU'(v), rounded once to out_dtype; v is the stored pre-activation."""
    return round_to(np.asarray(grad, dtype=np.float64) * gelu_erf_grad(v), out_dtype)


def dgelu_bgrad(grad, v, out_dtype: str = "bf16"):
    """(dv rounded to out_dtype, db = Σ_m grad·GELU'(v) in float64, before any rounding)."""
    exact = np.asarray(grad, dtype=np.float64) * gelu_erf_grad(v)
    return round_to(exact, out_dtype), bias_grad(exact)


# ---------------------------------------------------------------- LayerNorm after the tail
def layer_norm(x, gamma, beta, eps: float, out_dtype: str = "f32"):
    """z = (x − μ)/√(σ² + ε)·γ + β over the last dimension, rounded once to out_dtype.

    [mhc] §3.2: LayerNorm reduces a row to its mean and variance, then normalises
    the row; the BERT tail (bias → GELU → + residual → × 0.5) is followed by it.
    μ = mean over the row, σ² = mean((x − μ)²) (the population variance), in fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    z = (x - mu) / np.sqrt(var + float(eps)) * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)
    return round_to(z, out_dtype)
