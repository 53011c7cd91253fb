"""Seeded synthetic inputs for the fused linear layer y = act(A·Wᵀ + bias).

This module is shared by the tests, ``bench.py`` and ``__graft_entry__.smoke``.
It only draws random numbers and rounds them to the storage dtype; it holds
none of the layer's arithmetic (no GEMM, bias, activation or mask), so the
oracle and the CUDA path stay independent of each other.

Recipe (identical for every consumer):
  * ``torch.Generator('cpu').manual_seed(seed)``; every tensor is drawn in
    fp32 in the order listed by its workload, then rounded once (RNE) to its
    storage dtype with ``Tensor.to``.  The *rounded* tensors are what both the
    oracle and the kernels consume.
  * Distributions and shapes follow the five synthetic workloads of the fused
    linear layer (uniform[0,1) for the small RELU_BIAS case from the
    cuBLASLt epilog page's code example, N(0,1) for the Linear+GELU unit test
    of the zwxr.cn Linear+GELU fusion page §3.2, N(0,0.02²) weights for the
    GeGLU MLP of the "PyTorch MLP 核算子融合" page, N(0,1)/64 for the large
    training / BERT-tail shapes).

Nothing here touches a GPU; callers move tensors with ``.to(device)``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

__all__ = [
    "Workload", "WORKLOADS", "get", "make_inputs", "ragged_linear_inputs",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape/dtype description of one synthetic workload.

    ``kind`` selects the call pattern:
      * ``linear``  — one fused call ``out = epi(A·Wᵀ + bias)`` (or ``A·B`` when
        ``b_major`` is 1, i.e. B stored [K,N]).
      * ``geglu``   — dual gate/up call writing h, then the down projection.
      * ``relu_aux``— RELU_AUX_BIAS forward plus the dReLU backward step.
    """
    name: str
    kind: str
    M: int
    N: int
    K: int
    dtype: str               # operand storage dtype: "f16" | "bf16" | "f32"
    epilogue: str            # NONE|BIAS|RELU_BIAS|RELU_AUX_BIAS|GELU_BIAS|GELU_TANH_BIAS|GEGLU_TANH
    out_dtype: str
    bias_dtype: Optional[str] = None
    bias_axis: int = 0       # 0: bias[n] (per output feature of A·Wᵀ); 1: bias[m]
    b_major: int = 0         # 0: W is [N,K] (K contiguous); 1: B is [K,N] (N contiguous)
    residual: bool = False
    scale: float = 1.0
    dist: str = "normal"     # "uniform01" | "normal" | "normal/64"
    w_std: float = 1.0       # only used by the GeGLU weights
    compute: str = "32F"     # "32F" (fp16/bf16 in, fp32 acc) | "32F_3XTF32" (fp32 in)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs (2·M·N·K per GEMM; epilogue flops are not counted)."""
        if self.kind == "geglu":
            return 2.0 * self.M * (2 * self.N) * self.K + 2.0 * self.M * self.K * self.N
        return 2.0 * self.M * self.N * self.K


_TD = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _TD[name]


def _tail(M):
    return Workload(name=f"tail_m{M}", kind="linear", M=M, N=4096, K=4096, dtype="bf16",
                    epilogue="GELU_BIAS", out_dtype="f32", bias_dtype="bf16",
                    residual=True, scale=0.5, dist="normal/64")


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    # y = relu(W·x + b): W fp16 [100,784] is A (M=100), x fp16 [784,256] is B stored [K,N].
    Workload(name="relu_bias_100x256x784", kind="linear", M=100, N=256, K=784, dtype="f16",
             epilogue="RELU_BIAS", out_dtype="f32", bias_dtype="f32", bias_axis=1, b_major=1,
             dist="uniform01"),
    Workload(name="linear_gelu_f32_1024x3072x768", kind="linear", M=1024, N=3072, K=768,
             dtype="f32", epilogue="GELU_BIAS", out_dtype="f32", bias_dtype="f32",
             compute="32F_3XTF32"),
    Workload(name="linear_gelu_tanh_bf16_1024x3072x768", kind="linear", M=1024, N=3072, K=768,
             dtype="bf16", epilogue="GELU_TANH_BIAS", out_dtype="bf16", bias_dtype="bf16"),
    # GeGLU MLP: x [8192,768]; N here is the intermediate width (h is [8192,3072]).
    Workload(name="geglu_mlp_8192x3072x768", kind="geglu", M=8192, N=3072, K=768, dtype="bf16",
             epilogue="GEGLU_TANH", out_dtype="bf16", w_std=0.02),
    Workload(name="relu_aux_4096", kind="relu_aux", M=4096, N=4096, K=4096, dtype="bf16",
             epilogue="RELU_AUX_BIAS", out_dtype="bf16", bias_dtype="bf16", dist="normal/64"),
    _tail(32), _tail(128), _tail(512), _tail(2048),
]}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _draw(g: torch.Generator, shape, dist: str, std: float = 1.0) -> torch.Tensor:
    if dist == "uniform01":
        return torch.rand(*shape, generator=g, dtype=torch.float32)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if dist == "normal/64":
        return t / 64.0
    return t * std if std != 1.0 else t


def make_inputs(w: Workload, seed: int = 0, M: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """CPU tensors for workload ``w`` (rounded to storage dtypes).

    ``M`` overrides the row count (used to draw a bounded prefix for CPU
    timing); rows beyond the requested M are never drawn, so a prefix drawn
    with a smaller M is NOT the prefix of the full tensor — callers that want
    a sample of the full workload slice the full tensors instead.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    M = w.M if M is None else M
    td = _TD[w.dtype]
    out: Dict[str, torch.Tensor] = {}
    if w.kind == "geglu":
        out["x"] = _draw(g, (M, w.K), "normal").to(td)
        out["Wg"] = _draw(g, (w.N, w.K), "normal", w.w_std).to(td)
        out["Wu"] = _draw(g, (w.N, w.K), "normal", w.w_std).to(td)
        out["Wd"] = _draw(g, (w.K, w.N), "normal", w.w_std).to(td)
        return out
    if w.b_major:
        out["A"] = _draw(g, (M, w.K), w.dist).to(td)          # W of y = W·x
        out["B"] = _draw(g, (w.K, w.N), w.dist).to(td)        # x of y = W·x, stored [K,N]
    else:
        out["A"] = _draw(g, (M, w.K), w.dist).to(td)
        out["W"] = _draw(g, (w.N, w.K), w.dist).to(td)
    if w.bias_dtype is not None:
        blen = M if w.bias_axis == 1 else w.N
        out["bias"] = _draw(g, (blen,), w.dist).to(_TD[w.bias_dtype])
    if w.residual:
        out["residual"] = _draw(g, (M, w.N), w.dist).to(td)
    if w.kind == "relu_aux":
        out["grad"] = _draw(g, (M, w.N), "normal").to(td)
    return out


def ragged_linear_inputs(M: int, N: int, K: int, dtype: str, seed: int, *,
                         bias_dtype: Optional[str] = None, bias_axis: int = 0,
                         residual: bool = False, b_major: int = 0, dual: bool = False,
                         pad: int = 8, dist: str = "normal") -> Dict[str, torch.Tensor]:
    """Inputs for small ragged shapes used by the parity tests.

    Leading dimensions are padded up to a multiple of ``pad`` elements (TMA
    needs 16-byte aligned row pitches) while the logical extents stay ragged;
    the tensors returned are the padded storage and the padding holds random
    garbage that a correct kernel never reads.  ``dual`` draws a stacked
    [2N, K] weight for the gate/up GEMM.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    td = _TD[dtype]

    def padded(rows, cols):
        ld = -(-cols // pad) * pad
        return _draw(g, (rows, ld), dist).to(td)

    out: Dict[str, torch.Tensor] = {}
    out["A"] = padded(M, K)
    if b_major:
        out["B"] = padded(K, N)
    else:
        out["W"] = padded(2 * N if dual else N, K)
    if bias_dtype is not None:
        out["bias"] = _draw(g, (M if bias_axis == 1 else N,), dist).to(_TD[bias_dtype])
    if residual:
        out["residual"] = padded(M, N)
    return out


def all_names() -> List[str]:
    return list(WORKLOADS)
