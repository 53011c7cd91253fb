"""The seeded input generator shared by the oracle tests, the GPU parity tests and the bench.

Checks the recipe the tests rely on: the same seed gives the same tensors, every tensor
already holds values of its storage type (rounded once), shapes and distributions are
those of each workload, and ragged inputs keep 16-byte row pitches.
"""
from __future__ import annotations

import math

import pytest
import torch

import workloads

_ES = {"f16": 2, "bf16": 2, "f32": 4}


@pytest.mark.parametrize("name", ["relu_bias_100x256x784", "linear_gelu_f32_1024x3072x768", "tail_m32"])
def test_same_seed_same_tensors(name):
    w = workloads.get(name)
    a, b = workloads.make_inputs(w, 3), workloads.make_inputs(w, 3)
    c = workloads.make_inputs(w, 4)
    assert a.keys() == b.keys()
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert not torch.equal(a["A"], c["A"])


def test_shapes_dtypes_and_distributions_of_every_workload():
    for name in workloads.all_names():
        w = workloads.get(name)
        if w.M * w.K > 4096 * 4096 and w.kind != "geglu":
            continue
        t = workloads.make_inputs(w, 0)
        td = workloads.torch_dtype(w.dtype)
        if w.kind == "geglu":
            assert t["x"].shape == (w.M, w.K) and t["Wg"].shape == (w.N, w.K)
            assert t["Wu"].shape == (w.N, w.K) and t["Wd"].shape == (w.K, w.N)
            # N(0, 0.02²) weights
            assert abs(float(t["Wg"].float().std()) - w.w_std) < 0.05 * w.w_std
            continue
        A = t["A"]
        Wt = t["B"] if w.b_major else t["W"]
        assert A.shape == (w.M, w.K) and A.dtype == td
        assert Wt.shape == ((w.K, w.N) if w.b_major else (w.N, w.K)) and Wt.dtype == td
        if w.bias_dtype:
            assert t["bias"].shape == ((w.M,) if w.bias_axis else (w.N,))
            assert t["bias"].dtype == workloads.torch_dtype(w.bias_dtype)
        if w.residual:
            assert t["residual"].shape == (w.M, w.N)
        if w.kind == "relu_aux":
            assert t["grad"].shape == (w.M, w.N)
        a = A.float()
        if w.dist == "uniform01":
            # U[0,1) drawn in fp32; rounding to fp16 can carry the largest draws up to 1.0
            assert float(a.min()) >= 0.0 and float(a.max()) <= 1.0
            assert abs(float(a.mean()) - 0.5) < 0.01
        elif w.dist == "normal/64":
            assert abs(float(a.std()) - 1 / 64) < 0.05 / 64
        else:
            assert abs(float(a.std()) - 1.0) < 0.05


def test_values_are_already_in_the_storage_type():
    # rounding once more to the storage type changes nothing
    for name in ["relu_bias_100x256x784", "linear_gelu_tanh_bf16_1024x3072x768", "tail_m128"]:
        w = workloads.get(name)
        for k, v in workloads.make_inputs(w, 1).items():
            assert torch.equal(v.to(torch.float64).to(v.dtype), v), (name, k)


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_ragged_inputs_keep_16_byte_pitches(dtype):
    M, N, K = 37, 77, 45
    t = workloads.ragged_linear_inputs(M, N, K, dtype, 0, bias_dtype="f32", residual=True, pad=16 // _ES[dtype])
    for key, rows, cols in [("A", M, K), ("W", N, K), ("residual", M, N)]:
        x = t[key]
        assert x.shape[0] == rows and x.shape[1] >= cols
        assert (x.shape[1] * _ES[dtype]) % 16 == 0, (key, x.shape)
    assert t["bias"].shape == (N,)
    d = workloads.ragged_linear_inputs(M, N, K, dtype, 0, dual=True, pad=16 // _ES[dtype])
    assert d["W"].shape[0] == 2 * N


def test_flops_count_every_gemm():
    w = workloads.get("geglu_mlp_8192x3072x768")
    assert w.flops == 2 * w.M * (2 * w.N) * w.K + 2 * w.M * w.K * w.N
    t = workloads.get("tail_m32")
    assert t.flops == 2 * 32 * 4096 * 4096
    assert math.isclose(workloads.get("relu_aux_4096").flops, 2 * 4096 ** 3)
