"""Oracle for the fused linear layer — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct CPU statement (numpy/scipy, float64) of what
the fused linear layer computes.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm may import it.  The CUDA
product path never imports, links or calls anything here, and nothing here
imports the product package: the two share no code.

Sources (four web pages on GEMM epilogue fusion; cited by title and section):
  [epilog]  "通过 cuBLASLt 的 epilog 机制实现单内核偏置融合：参数配置与性能收益"
            (blog.hotdry.top) — Matmul → plan(epilog, epilog_inputs{bias}) →
            execute; RELU_BIAS / GELU_BIAS / RELU_AUX_BIAS; bias matches the
            result's first (output-feature) dimension; FP32 compute type.
  [gelu]    zwxr.cn/news/294525, "Linear+GELU 算子融合" — §1 GELU(x)=x·Φ(x)
            =0.5x[1+erf(x/√2)], §2.1 the PyTorch erf form, §2.2.2 the tanh form
            with 0.044715 and √(2/π), §3.2 the Linear+GELU unit test.
  [mlp]     "PyTorch MLP 核算子融合：從 nn.Linear 到 Fused MLP"
            (wiki-fongyasong) — addmm(bias,x,weight) = x @ weight.T + bias;
            the GeGLU MLP h = gelu(gate_proj(x)) * up_proj(x), then down_proj.
  [mhc]     mhpn.cn/news/2504128, "mHC 融合" — §2.2 elementwise chains
            (bias add, residual add, multiply by a constant), §4.2 the fused
            BiasGELU kernel with the constant 0.79788456.

Every function below is pinned by ``tests/test_oracle.py`` against brute
force, closed forms, identities or an independent library routine; none is
"parity unpinned".
"""
from .fused_linear import (  # noqa: F401
    gemm, add_bias, relu, gelu_erf, gelu_tanh, activation, relu_aux_mask,
    residual_scale, round_to, fused_linear, geglu_h, geglu_mlp, drelu,
    bias_grad, drelu_bgrad, gelu_erf_grad, dgelu, dgelu_bgrad, gelu_sigmoid, layer_norm,
    GELU_TANH_C, GELU_TANH_A, GELU_SIGMOID_K,
)
