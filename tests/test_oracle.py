"""CPU tests: the oracle against its pins, and planted mistakes that the pins must catch.

A mutation test replaces one oracle function with a plausible mistake (a
dropped term, a wrong sign or index, a transposed operand, a wrong constant)
in a throw-away namespace on the CPU and checks that at least one pin fails.
"""
from __future__ import annotations

import math
import types

import numpy as np
import pytest
from scipy.special import erf

import oracle
from tests import oracle_pins as P

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def _namespace(**over):
    ns = types.SimpleNamespace(**{k: getattr(oracle, k) for k in oracle.__all__}) \
        if hasattr(oracle, "__all__") else None
    if ns is None:
        names = ["gemm", "add_bias", "relu", "gelu_erf", "gelu_tanh", "activation", "relu_aux_mask",
                 "residual_scale", "round_to", "fused_linear", "geglu_h", "geglu_mlp", "drelu",
                 "bias_grad", "drelu_bgrad", "gelu_erf_grad", "dgelu", "dgelu_bgrad", "gelu_sigmoid", "layer_norm"]
        ns = types.SimpleNamespace(**{k: getattr(oracle, k) for k in names})
    for k, v in over.items():
        setattr(ns, k, v)

    # Rebind the composite functions so that they use the (possibly mutated) parts.
    def fused_linear(A, W, bias=None, *, epilogue, out_dtype, bias_axis=0, b_major=0,
                     residual=None, scale=1.0):
        v = ns.gemm(A, W, b_major)
        if bias is not None and epilogue != "NONE":
            v = ns.add_bias(v, bias, bias_axis)
        a = ns.activation(v, epilogue)
        y = ns.residual_scale(a, residual, scale)
        aux = None
        if epilogue == "RELU_AUX_BIAS":
            aux = ns.relu_aux_mask(v)
        elif epilogue == "GELU_AUX_BIAS":
            aux = ns.round_to(v, out_dtype)
        return ns.round_to(y, out_dtype), aux, v

    def activation(v, kind):
        if kind in ("NONE", "BIAS"):
            return v
        if kind in ("RELU_BIAS", "RELU_AUX_BIAS", "RELU"):
            return ns.relu(v)
        if kind in ("GELU_BIAS", "GELU_AUX_BIAS", "GELU"):
            return ns.gelu_erf(v)
        if kind in ("GELU_SIGMOID_BIAS", "GELU_SIGMOID"):
            return ns.gelu_sigmoid(v)
        return ns.gelu_tanh(v)

    def drelu_bgrad(grad, aux, N, out_dtype="bf16"):
        dv = ns.drelu(grad, aux, N, out_dtype)
        return dv, ns.bias_grad(dv)

    def dgelu(grad, v, out_dtype="bf16"):
        return ns.round_to(np.asarray(grad, float) * ns.gelu_erf_grad(v), out_dtype)

    def dgelu_bgrad(grad, v, out_dtype="bf16"):
        exact = np.asarray(grad, float) * ns.gelu_erf_grad(v)
        return ns.round_to(exact, out_dtype), ns.bias_grad(exact)

    def geglu_h(x, Wg, Wu, out_dtype="bf16"):
        return ns.round_to(ns.gelu_tanh(ns.gemm(x, Wg)) * ns.gemm(x, Wu), out_dtype)

    def geglu_mlp(x, Wg, Wu, Wd, out_dtype="bf16"):
        h = ns.geglu_h(x, Wg, Wu, out_dtype)
        return h, ns.round_to(ns.gemm(h, Wd), out_dtype)

    for name, f in [("fused_linear", fused_linear), ("activation", activation),
                    ("geglu_h", geglu_h), ("geglu_mlp", geglu_mlp), ("drelu_bgrad", drelu_bgrad),
                    ("dgelu", dgelu), ("dgelu_bgrad", dgelu_bgrad)]:
        if name not in over:
            setattr(ns, name, f)
    return ns


def _gemm_transposed_w(A, W, b_major=0):
    A = np.asarray(A, float)
    W = np.asarray(W, float)
    if b_major:
        return A @ W
    return A @ W.reshape(W.shape[1], W.shape[0]).T if W.shape[0] != W.shape[1] else A @ W


def _mask_msb_first(v):
    M, N = v.shape
    out = np.zeros((M, (N + 31) // 32), dtype=np.uint64)
    for n in range(N):
        out[:, n // 32] |= (v[:, n] > 0).astype(np.uint64) << np.uint64(31 - n % 32)
    return out.astype(np.uint32)


def _mask_ge(v):
    M, N = v.shape
    out = np.zeros((M, (N + 31) // 32), dtype=np.uint64)
    for n in range(N):
        out[:, n // 32] |= (v[:, n] >= 0).astype(np.uint64) << np.uint64(n % 32)
    return out.astype(np.uint32)


MUTANTS = {
    "gemm_transposed_operand": dict(gemm=_gemm_transposed_w),
    "gemm_drops_last_k": dict(gemm=lambda A, W, b_major=0: (np.asarray(A, float)[:, :-1] @ (
        np.asarray(W, float)[:-1, :] if b_major else np.asarray(W, float)[:, :-1].T))),
    "bias_wrong_axis": dict(add_bias=lambda acc, b, axis=0: acc + (np.asarray(b)[:, None] if axis == 0 else np.asarray(b)[None, :])
                            if acc.shape[0] == acc.shape[1] else acc + np.resize(np.asarray(b, float), acc.shape)),
    "bias_dropped": dict(add_bias=lambda acc, b, axis=0: acc),
    "gelu_no_half": dict(gelu_erf=lambda v: v * (1.0 + erf(np.asarray(v) / math.sqrt(2.0)))),
    "gelu_sign": dict(gelu_erf=lambda v: 0.5 * np.asarray(v) * (1.0 - erf(np.asarray(v) / math.sqrt(2.0)))),
    "gelu_no_sqrt2": dict(gelu_erf=lambda v: 0.5 * np.asarray(v) * (1.0 + erf(np.asarray(v)))),
    "gelu_tanh_wrong_cubic": dict(gelu_tanh=lambda v: 0.5 * np.asarray(v) * (1.0 + np.tanh(
        math.sqrt(2 / math.pi) * (np.asarray(v) + 0.0447 * np.asarray(v) ** 3)))),
    "gelu_tanh_is_erf": dict(gelu_tanh=lambda v: oracle.gelu_erf(v)),
    "gelu_tanh_no_sqrt": dict(gelu_tanh=lambda v: 0.5 * np.asarray(v) * (1.0 + np.tanh(
        (2 / math.pi) * (np.asarray(v) + 0.044715 * np.asarray(v) ** 3)))),
    "relu_leaky": dict(relu=lambda v: np.where(np.asarray(v) > 0, v, 0.01 * np.asarray(v))),
    "mask_msb_first": dict(relu_aux_mask=_mask_msb_first),
    "mask_ge_zero": dict(relu_aux_mask=_mask_ge),
    "residual_after_scale": dict(residual_scale=lambda a, r, s: a * s + (0 if r is None else np.asarray(r, float))),
    "residual_dropped": dict(residual_scale=lambda a, r, s: a * s),
    "round_truncates": dict(round_to=lambda x, d: (np.trunc(np.asarray(x, float) * 256) / 256) if d == "bf16"
                            else oracle.round_to(x, d)),
    "bias_grad_over_columns": dict(bias_grad=lambda dv: np.asarray(dv, float).sum(axis=1)[:np.asarray(dv).shape[1]]
                                   if np.asarray(dv).shape[0] >= np.asarray(dv).shape[1]
                                   else np.resize(np.asarray(dv, float).sum(axis=1), np.asarray(dv).shape[1])),
    "bias_grad_mean": dict(bias_grad=lambda dv: np.asarray(dv, float).mean(axis=0)),
    "gelu_grad_drops_vphi": dict(gelu_erf_grad=lambda v: 0.5 * (1.0 + erf(np.asarray(v, float) / math.sqrt(2.0)))),
    "gelu_grad_phi_sign": dict(gelu_erf_grad=lambda v: 0.5 * (1.0 + erf(np.asarray(v, float) / math.sqrt(2.0)))
                               - np.asarray(v, float) * np.exp(-0.5 * np.asarray(v, float) ** 2) / math.sqrt(2 * math.pi)),
    "gelu_grad_no_half_exponent": dict(gelu_erf_grad=lambda v: 0.5 * (1.0 + erf(np.asarray(v, float) / math.sqrt(2.0)))
                                       + np.asarray(v, float) * np.exp(-np.asarray(v, float) ** 2) / math.sqrt(2 * math.pi)),
    "gelu_sigmoid_slope_one": dict(gelu_sigmoid=lambda v: np.asarray(v, float) / (1.0 + np.exp(-np.asarray(v, float)))),
    "gelu_sigmoid_sign": dict(gelu_sigmoid=lambda v: np.asarray(v, float) / (1.0 + np.exp(1.702 * np.asarray(v, float)))),
    "layer_norm_sample_variance": dict(layer_norm=lambda x, g, b, eps, od="f32": oracle.round_to(
        (np.asarray(x, float) - np.asarray(x, float).mean(-1, keepdims=True))
        / np.sqrt(np.asarray(x, float).var(-1, ddof=1, keepdims=True) + eps) * g + b, od)),
    "layer_norm_eps_outside_sqrt": dict(layer_norm=lambda x, g, b, eps, od="f32": oracle.round_to(
        (np.asarray(x, float) - np.asarray(x, float).mean(-1, keepdims=True))
        / (np.sqrt(np.asarray(x, float).var(-1, keepdims=True)) + eps) * g + b, od)),
    "layer_norm_no_beta": dict(layer_norm=lambda x, g, b, eps, od="f32": oracle.round_to(
        (np.asarray(x, float) - np.asarray(x, float).mean(-1, keepdims=True))
        / np.sqrt(np.asarray(x, float).var(-1, keepdims=True) + eps) * g, od)),
    "drelu_inverted": dict(drelu=lambda grad, aux, N, od="bf16": oracle.round_to(
        np.asarray(grad, float)[:, :N] - oracle.drelu(grad, aux, N, od), od)),
    # the down projection of the unrounded h (h kept in fp64 instead of the bf16 tensor)
    "geglu_mlp_skips_h_rounding": dict(geglu_mlp=lambda x, Wg, Wu, Wd, od="bf16": (
        oracle.geglu_h(x, Wg, Wu, od),
        oracle.round_to(oracle.gemm(oracle.gelu_tanh(oracle.gemm(x, Wg)) * oracle.gemm(x, Wu), Wd), od))),
    # Wd read as [in, out] (h @ Wd in place of h @ Wdᵀ)
    "geglu_mlp_transposed_wd": dict(geglu_mlp=lambda x, Wg, Wu, Wd, od="bf16": (
        oracle.geglu_h(x, Wg, Wu, od),
        oracle.round_to(oracle.gemm(oracle.geglu_h(x, Wg, Wu, od), Wd, b_major=1), od))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    ns = _namespace(**MUTANTS[name])
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(ns)
        except AssertionError:
            failed.append(pin.__name__)
        except Exception as e:  # shape errors etc. also count as caught
            failed.append(f"{pin.__name__}:{type(e).__name__}")
    assert failed, f"no pin caught the planted mistake {name}"


def test_unmutated_namespace_passes_all_pins():
    ns = _namespace()
    for pin in P.ALL_PINS:
        pin(ns)
