"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small and ragged shapes are compared element by element over the whole
output; the full-size synthetic workloads are compared on sampled rows that
the oracle computes one by one (the GPU computes everything, in the launch
configuration the benchmark times).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import gemm_bias_activation_tcgen05_b200 as m
    return m


def _linear_case(fl, M, N, K, *, dtype="bf16", epilogue="GELU_BIAS", out_dtype="bf16", bias_axis=0,
                 residual=False, scale=1.0, b_major=0, seed=0, bias_dtype=None, unfused=False, schedule="auto",
                 bias_offset=0):
    bias_dtype = bias_dtype or ("f32" if dtype == "f32" else dtype)
    has_bias = epilogue not in ("NONE",)
    inp = workloads.ragged_linear_inputs(M, N, K, dtype, seed, bias_dtype=bias_dtype if has_bias else None,
                                         bias_axis=bias_axis, residual=residual, b_major=b_major)
    W = inp["B"] if b_major else inp["W"]
    got = P.run_linear(fl, M=M, N=N, K=K, dtype=dtype, epilogue=epilogue, out_dtype=out_dtype, A=inp["A"],
                       W=W, bias=inp.get("bias"), bias_dtype=bias_dtype, bias_axis=bias_axis, b_major=b_major,
                       residual=inp.get("residual"), residual_dtype=dtype, scale=scale, unfused=unfused,
                       schedule=schedule, bias_offset=bias_offset)
    y, aux, v, absdot = P.oracle_linear(A=inp["A"], W=W, bias=inp.get("bias"), bias_axis=bias_axis,
                                        b_major=b_major, residual=inp.get("residual"), scale=scale,
                                        epilogue=epilogue, out_dtype=out_dtype, M=M, N=N, K=K)
    what = f"{epilogue} {dtype}->{out_dtype} M{M} N{N} K{K} bias+{bias_offset} info={got['info']}"
    P.check_close(got["out"], y, out_dtype, absdot, what)
    if epilogue == "RELU_AUX_BIAS":
        margin = None
        if unfused:
            # the twin rounds acc = A·Wᵀ to the output dtype before the bias step
            acc = v - (P.to64(inp["bias"])[None, :] if bias_axis == 0 else P.to64(inp["bias"])[:, None])
            margin = P.ULP_REL[out_dtype] * (np.abs(acc) + np.abs(v))
        P.check_mask(got["aux"], v, N, what, margin)
    return got


def test_single_tile_plain_gemm(fl):
    _linear_case(fl, 128, 128, 64, epilogue="NONE", out_dtype="f32")


def test_multi_kblock_multi_tile(fl):
    _linear_case(fl, 256, 512, 320, epilogue="NONE", out_dtype="f32")


@pytest.mark.parametrize("out_dtype", ["bf16", "f32", "f16"])
@pytest.mark.parametrize("epilogue", ["NONE", "BIAS", "RELU_BIAS", "RELU_AUX_BIAS", "GELU_BIAS", "GELU_TANH_BIAS",
                                      "GELU_SIGMOID_BIAS"])
def test_epilogues_ragged(fl, epilogue, out_dtype):
    # ragged in every dimension: M, N not tile multiples, K not a multiple of 64
    _linear_case(fl, 300, 520, 200, epilogue=epilogue, out_dtype=out_dtype, seed=11)


@pytest.mark.parametrize("epilogue,out_dtype,dtype", [("RELU_AUX_BIAS", "bf16", "bf16"),
                                                       ("GELU_TANH_BIAS", "f16", "f16"),
                                                       ("GELU_BIAS", "f32", "bf16")])
def test_192_wide_tiles(fl, epilogue, out_dtype, dtype):
    # 1000 x 2568: 192-wide pair tiles are the cheapest (56 tiles in one round, against 84
    # 128-wide ones).  With a 16-bit output each warp's last 32 columns of a tile go out by
    # direct stores instead of TMA, and the last column tile (72 wide) ends inside those 32
    import gemm_bias_activation_tcgen05_b200 as m
    info = m.fl_plan_preview(1000, 2568, 200, dtype, kind=epilogue, out_dtype=out_dtype)
    assert info["tile_n"] == 192 and info["cta_pair"] == 1, info
    _linear_case(fl, 1000, 2568, 200, dtype=dtype, epilogue=epilogue, out_dtype=out_dtype, seed=17,
                 bias_dtype="f32" if out_dtype == "f32" else dtype)


@pytest.mark.parametrize("bias_dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("bias_offset", [0, 1, 8])
@pytest.mark.parametrize("M,epilogue", [(200, "GELU_TANH_BIAS"), (100, "RELU_AUX_BIAS")])
def test_bias_alignment(fl, bias_dtype, bias_offset, M, epilogue):
    # a per-column bias on and off the 16-byte grid, over whole and ragged 32-column
    # blocks (N = 300), on CTA pairs and single CTAs
    _linear_case(fl, M, 300, 136, epilogue=epilogue, out_dtype="bf16", bias_dtype=bias_dtype,
                 bias_offset=bias_offset, seed=21)


def test_fp16_operands(fl):
    _linear_case(fl, 257, 264, 136, dtype="f16", epilogue="GELU_TANH_BIAS", out_dtype="f16", bias_dtype="f16")


def test_bias_per_row(fl):
    _linear_case(fl, 200, 384, 96, epilogue="RELU_BIAS", out_dtype="f32", bias_axis=1, bias_dtype="f32")


def test_residual_and_scale(fl):
    _linear_case(fl, 384, 640, 256, epilogue="GELU_BIAS", out_dtype="f32", residual=True, scale=0.5)


@pytest.mark.parametrize("M,N,K", [(100, 256, 784), (129, 200, 72), (256, 512, 128)])
def test_b_stored_k_by_n(fl, M, N, K):
    _linear_case(fl, M, N, K, dtype="f16", epilogue="RELU_BIAS", out_dtype="f32", bias_axis=1,
                 bias_dtype="f32", b_major=1)


@pytest.mark.parametrize("M", [1, 5, 32, 77, 128])
def test_small_m_swap_split_k(fl, M):
    got = _linear_case(fl, M, 1000, 1000, epilogue="GELU_BIAS", out_dtype="f32", residual=True, scale=0.5,
                       seed=M)
    assert got["info"]["swap_ab"] == 1


@pytest.mark.parametrize("M,dtype", [(9, "bf16"), (100, "f16"), (200, "f32")])
def test_sigmoid_gelu_layouts(fl, M, dtype):
    # swap-AB (M <= 128, 16-bit), and the 3xTF32 pair path for fp32 operands
    got = _linear_case(fl, M, 1000, 520, dtype=dtype, epilogue="GELU_SIGMOID_BIAS", out_dtype="f32", seed=M)
    assert got["info"]["swap_ab"] == (1 if dtype != "f32" else 0)


@pytest.mark.parametrize("M", [16, 100])
def test_small_m_relu_aux(fl, M):
    _linear_case(fl, M, 520, 264, epilogue="RELU_AUX_BIAS", out_dtype="bf16", seed=3)


def test_k_zero_is_bias_only(fl):
    _linear_case(fl, 130, 136, 0, epilogue="GELU_BIAS", out_dtype="f32", residual=True, scale=0.5)


@pytest.mark.parametrize("M,N,K", [(200, 300, 136), (128, 128, 64), (257, 136, 768)])
def test_geglu_dual(fl, M, N, K):
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 5, dual=True)
    A, W = inp["A"], inp["W"]
    ldh = -(-N // 8) * 8
    got = P.run_linear(fl, M=M, N=N, K=K, dtype="bf16", epilogue="GEGLU_TANH", out_dtype="bf16", A=A, W=W)
    a = P.to64(A)[:, :K]
    w = P.to64(W)
    Wg, Wu = w[:N, :K], w[N:2 * N, :K]
    h = oracle.geglu_h(a, Wg, Wu, "bf16")
    g = oracle.gemm(a, Wg)
    u = oracle.gemm(a, Wu)
    absdot = float((oracle.gemm(np.abs(a), np.abs(Wg)) * np.abs(u) * 1.2
                    + oracle.gemm(np.abs(a), np.abs(Wu)) * np.abs(oracle.gelu_tanh(g))).max())
    assert ldh >= N
    P.check_close(got["out"], h, "bf16", absdot, f"geglu {M}x{N}x{K}")


@pytest.mark.parametrize("epilogue", ["RELU_AUX_BIAS", "GELU_TANH_BIAS", "NONE", "GELU_SIGMOID_BIAS"])
def test_unfused_twin(fl, epilogue):
    got = _linear_case(fl, 256, 384, 192, epilogue=epilogue, out_dtype="bf16", unfused=True, seed=7)
    assert got["info"]["launches_per_execute"] >= 1


def test_unfused_residual_f32(fl):
    _linear_case(fl, 200, 264, 128, epilogue="GELU_BIAS", out_dtype="f32", residual=True, scale=0.5,
                 unfused=True)


@pytest.mark.parametrize("M,out_dtype", [(5, "f32"), (77, "f32"), (128, "f32"), (40, "bf16")])
def test_unfused_twin_small_m(fl, M, out_dtype):
    # M <= 128: the twin's bare GEMM takes the swap-AB layout with split-K, then the
    # bias, GELU, residual and scale steps run as separate kernels
    got = _linear_case(fl, M, 1000, 1000, epilogue="GELU_BIAS", out_dtype=out_dtype, residual=True, scale=0.5,
                       unfused=True, seed=40 + M)
    assert got["info"]["launches_per_execute"] == 5


@pytest.mark.parametrize("M,N,K", [(200, 300, 136), (77, 264, 200), (257, 136, 768)])
def test_unfused_twin_geglu(fl, M, N, K):
    # the twin of GEGLU_TANH: the bare dual GEMM writes [g | u] ([M, 2N]) to an
    # intermediate in the output type, then one kernel forms gelu_tanh(g)·u
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 9, dual=True)
    A, W = inp["A"], inp["W"]
    got = P.run_linear(fl, M=M, N=N, K=K, dtype="bf16", epilogue="GEGLU_TANH", out_dtype="bf16", A=A, W=W,
                       unfused=True)
    assert got["info"]["launches_per_execute"] == 2
    a = P.to64(A)[:, :K]
    w = P.to64(W)
    Wg, Wu = w[:N, :K], w[N:2 * N, :K]
    h = oracle.geglu_h(a, Wg, Wu, "bf16")
    g = oracle.gemm(a, Wg)
    u = oracle.gemm(a, Wu)
    absdot = float((oracle.gemm(np.abs(a), np.abs(Wg)) * np.abs(u) * 1.2
                    + oracle.gemm(np.abs(a), np.abs(Wu)) * np.abs(oracle.gelu_tanh(g))).max())
    # g and u pass through the bf16 intermediate, as in the eager chain: one more rounding
    # of each (at most 2^-8 relative), which moves h by up to |GELU'(g)|·2^-8|g|·|u| +
    # |GELU(g)|·2^-8|u| (GELU' of the tanh form stays below 1.2); near g = -2 that alone can
    # exceed the contract's 2e-2·max(1, |h|), so the twin is held to the contract plus it
    err = np.abs(got["out"] - h)
    bound = P.contract_tol(h, "bf16") + 2.0 ** -8 * (1.2 * np.abs(g) + np.abs(oracle.gelu_tanh(g))) * np.abs(u)
    assert np.all(np.isfinite(got["out"]))
    assert (err <= bound).all(), f"geglu twin {M}x{N}x{K}: {(err > bound).sum()} elements, worst {err.max():.3e}"
    absdot += float((np.abs(g) * np.abs(u)).max()) * 2.0 ** -8 * 2 ** 14
    tight = 2.0 * P.ULP_REL["bf16"] * float(np.abs(h).max()) + 2.0 ** -14 * absdot
    assert err.max() <= tight, (err.max(), tight)


@pytest.mark.parametrize("M,N,dtype", [(64, 4096, "bf16"), (33, 1000, "bf16"), (7, 77, "f32"), (5, 40, "f16")])
def test_relu_backward(fl, M, N, dtype):
    g = torch.Generator().manual_seed(M * N)
    v = torch.randn(M, N, generator=g, dtype=torch.float64).numpy()
    aux = oracle.relu_aux_mask(v)
    grad = torch.randn(M, N, generator=g).to(P.TD[dtype])
    dgrad = grad.cuda()
    daux = torch.from_numpy(aux.view(np.int32)).cuda()
    dpre = P.poison((M, N), dtype)
    fl.fl_relu_backward(dgrad, daux, dpre, M, N, dtype)
    torch.cuda.synchronize()
    ref = oracle.drelu(P.to64(grad), aux, N, dtype)
    out = P.to64(dpre)
    assert np.array_equal(out, ref)
    # grad·0 keeps the sign of grad, as an IEEE multiply does
    assert np.array_equal(np.signbit(out), np.signbit(ref))


# ---------------------------------------------------------------- full-size workloads
def _run_workload_linear(fl, w, seed=0, rows=256):
    inp = workloads.make_inputs(w, seed)
    W = inp["B"] if w.b_major else inp["W"]
    got = P.run_linear(fl, M=w.M, N=w.N, K=w.K, dtype=w.dtype, epilogue=w.epilogue, out_dtype=w.out_dtype,
                       A=inp["A"], W=W, bias=inp.get("bias"), bias_dtype=w.bias_dtype or "bf16",
                       bias_axis=w.bias_axis, b_major=w.b_major, residual=inp.get("residual"),
                       residual_dtype=w.dtype, scale=w.scale, out_pad=1)
    sel = P.sample_rows(w.M, rows, seed) if w.M > rows else None
    y, aux, v, absdot = P.oracle_linear(A=inp["A"], W=W, bias=inp.get("bias"), bias_axis=w.bias_axis,
                                        b_major=w.b_major, residual=inp.get("residual"), scale=w.scale,
                                        epilogue=w.epilogue, out_dtype=w.out_dtype, M=w.M, N=w.N, K=w.K,
                                        rows=sel)
    out = got["out"] if sel is None else got["out"][sel]
    P.check_close(out, y, w.out_dtype, absdot, f"{w.name} seed {seed} info={got['info']}")
    if w.epilogue == "RELU_AUX_BIAS":
        aux_g = got["aux"] if sel is None else got["aux"][sel]
        P.check_mask(aux_g, v, w.N, w.name)
    return got, inp, sel, v


@pytest.mark.parametrize("M,N,K,epilogue,out_dtype", [(300, 520, 200, "GELU_BIAS", "f32"),
                                                       (130, 264, 100, "RELU_AUX_BIAS", "bf16"),
                                                       (64, 136, 36, "BIAS", "f32"),
                                                       (257, 384, 768, "GELU_TANH_BIAS", "f16")])
def test_fp32_operands_3xtf32(fl, M, N, K, epilogue, out_dtype):
    got = _linear_case(fl, M, N, K, dtype="f32", epilogue=epilogue, out_dtype=out_dtype, seed=13)
    assert got["info"]["swap_ab"] == 0
    # beyond one 128-row tile the 3xTF32 UMMA runs on CTA pairs
    assert got["info"]["cta_pair"] == (1 if M > 128 else 0)


@pytest.mark.parametrize("M", [64, 130])
def test_fp32_split_with_all_low_bits_set(fl, M):
    # Every operand word has its 13 low mantissa bits set, where truncating and
    # rounding an fp32 word to TF32 differ the most: the 3xTF32 split must still
    # be exact to about 2^-21 per product.  (K is short so that one wrong hi word,
    # an error near 2^-10 of a product, stands far above the bound.)
    N, K = 200, 24
    g = torch.Generator().manual_seed(M)

    def words(rows, cols):
        x = torch.randn(rows, cols, generator=g, dtype=torch.float32)
        b = x.view(torch.int32) | 0x1FFF
        return b.view(torch.float32).contiguous()

    A, W = words(M, K), words(N, K)
    got = P.run_linear(fl, M=M, N=N, K=K, dtype="f32", epilogue="NONE", out_dtype="f32", A=A, W=W)
    y, _, _, absdot = P.oracle_linear(A=A, W=W, epilogue="NONE", out_dtype="f32", M=M, N=N, K=K)
    P.check_close(got["out"], y, "f32", absdot, f"fp32 low bits M{M}")


def test_fp32_residual_scale(fl):
    _linear_case(fl, 200, 264, 132, dtype="f32", epilogue="GELU_BIAS", out_dtype="f32", residual=True, scale=0.5)


@pytest.mark.parametrize("name", ["relu_bias_100x256x784", "linear_gelu_f32_1024x3072x768",
                                  "linear_gelu_tanh_bf16_1024x3072x768",
                                  "tail_m32", "tail_m128", "tail_m512", "tail_m2048"])
def test_workload_linear(fl, name):
    _run_workload_linear(fl, workloads.get(name))


def test_workload_relu_aux_with_backward(fl):
    w = workloads.get("relu_aux_4096")
    got, inp, sel, v = _run_workload_linear(fl, w)
    # backward on the full mask the forward wrote
    aux = torch.from_numpy(got["aux"].view(np.int32)).cuda()
    grad = inp["grad"].cuda()
    dpre = P.poison((w.M, w.N), "bf16")
    fl.fl_relu_backward(grad, aux, dpre, w.M, w.N, "bf16")
    torch.cuda.synchronize()
    ref = oracle.drelu(P.to64(inp["grad"])[sel], got["aux"][sel], w.N, "bf16")
    assert np.array_equal(P.to64(dpre)[sel], ref)


def test_workload_geglu_mlp(fl):
    w = workloads.get("geglu_mlp_8192x3072x768")
    inp = workloads.make_inputs(w, 0)
    x, Wg, Wu, Wd = inp["x"], inp["Wg"], inp["Wu"], inp["Wd"]
    Wgu = torch.cat([Wg, Wu], 0)
    dx, dW, dWd = x.cuda(), Wgu.cuda(), Wd.cuda()
    h = P.poison((w.M, w.N), "bf16")
    y = P.poison((w.M, w.K), "bf16")
    up = fl.Plan(w.M, w.N, w.K, kind="GEGLU_TANH", out_dtype="bf16")
    down = fl.Plan(w.M, w.K, w.N, kind="NONE", out_dtype="bf16")
    try:
        up.execute(dx, dW, out=h)
        down.execute(h, dWd, out=y)
        assert up.check() == fl.FL_OK and down.check() == fl.FL_OK, fl.fl_last_error()
    finally:
        up.free()
        down.free()
    sel = P.sample_rows(w.M, 128, 0)
    a = P.to64(x)[sel]
    g = oracle.gemm(a, P.to64(Wg))
    u = oracle.gemm(a, P.to64(Wu))
    h_ref = oracle.round_to(oracle.gelu_tanh(g) * u, "bf16")
    h_got = P.to64(h)[sel]
    absdot_h = float((oracle.gemm(np.abs(a), np.abs(P.to64(Wg))) * np.abs(u) * 1.2
                      + oracle.gemm(np.abs(a), np.abs(P.to64(Wu))) * np.abs(oracle.gelu_tanh(g))).max())
    P.check_close(h_got, h_ref, "bf16", absdot_h, "geglu h")
    # y against the oracle's down projection of the GPU's own bf16 h (isolates the second GEMM)
    y_ref = oracle.round_to(oracle.gemm(h_got, P.to64(Wd)), "bf16")
    absdot_y = float(oracle.gemm(np.abs(h_got), np.abs(P.to64(Wd))).max())
    P.check_close(P.to64(y)[sel], y_ref, "bf16", absdot_y, "geglu down_proj")


@pytest.mark.parametrize("M,N,K,out_dtype", [(256, 300, 100, "bf16"), (200, 5, 7, "bf16"), (130, 301, 37, "f32"),
                                             (64, 250, 100, "f32"), (300, 263, 519, "f16")])
def test_ragged_k_and_row_tail_nan_padding(fl, M, N, K, out_dtype):
    """Row padding of every input is NaN: a kernel that reads past K (or past N of
    the residual) produces NaN; the output padding must keep its poison."""
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 21, bias_dtype="bf16", residual=True)
    A, W, R = inp["A"].clone(), inp["W"].clone(), inp["residual"].clone()
    A[:, K:] = float("nan")
    W[:, K:] = float("nan")
    R[:, N:] = float("nan")
    got = P.run_linear(fl, M=M, N=N, K=K, dtype="bf16", epilogue="GELU_TANH_BIAS", out_dtype=out_dtype, A=A, W=W,
                       bias=inp["bias"], residual=R, scale=0.5, out_pad=16)
    y, _, _, absdot = P.oracle_linear(A=A, W=W, bias=inp["bias"], residual=R, scale=0.5,
                                      epilogue="GELU_TANH_BIAS", out_dtype=out_dtype, M=M, N=N, K=K)
    P.check_close(got["out"], y, out_dtype, absdot, f"ragged nan-padded {M}x{N}x{K} {got['info']}")


# ---------------------------------------------------------------- stream-K (CTA pairs)
@pytest.mark.parametrize("M,N,K,epilogue,out_dtype", [
    (600, 1000, 1000, "GELU_BIAS", "f32"),      # 12 tiles x 8 K blocks on 74 pairs: up to 7 writers a tile
    (300, 520, 2000, "RELU_AUX_BIAS", "bf16"),  # ragged, mask through the stream-K sums
    (1000, 264, 4000, "GELU_TANH_BIAS", "bf16"),
    (257, 136, 768, "BIAS", "f16"),
])
def test_stream_k_ragged(fl, M, N, K, epilogue, out_dtype):
    got = _linear_case(fl, M, N, K, epilogue=epilogue, out_dtype=out_dtype, residual=epilogue == "GELU_BIAS",
                       scale=0.5 if epilogue == "GELU_BIAS" else 1.0, seed=M + N, schedule="stream_k")
    assert got["info"]["cta_pair"] == 1 and got["info"]["stream_k_tiles"] > 0, got["info"]
    # the same layer on whole tiles only
    dp = _linear_case(fl, M, N, K, epilogue=epilogue, out_dtype=out_dtype, residual=epilogue == "GELU_BIAS",
                      scale=0.5 if epilogue == "GELU_BIAS" else 1.0, seed=M + N, schedule="data_parallel")
    assert dp["info"]["stream_k_tiles"] == 0


def test_stream_k_geglu(fl):
    M, N, K = 1000, 520, 700
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 17, dual=True)
    A, W = inp["A"], inp["W"]
    got = P.run_linear(fl, M=M, N=N, K=K, dtype="bf16", epilogue="GEGLU_TANH", out_dtype="bf16", A=A, W=W,
                       schedule="stream_k")
    assert got["info"]["stream_k_tiles"] > 0, got["info"]
    a = P.to64(A)[:, :K]
    w = P.to64(W)
    Wg, Wu = w[:N, :K], w[N:2 * N, :K]
    g = oracle.gemm(a, Wg)
    u = oracle.gemm(a, Wu)
    absdot = float((oracle.gemm(np.abs(a), np.abs(Wg)) * np.abs(u) * 1.2
                    + oracle.gemm(np.abs(a), np.abs(Wu)) * np.abs(oracle.gelu_tanh(g))).max())
    P.check_close(got["out"], oracle.geglu_h(a, Wg, Wu, "bf16"), "bf16", absdot, f"stream-K geglu {got['info']}")


def test_stream_k_unfused_twin(fl):
    got = _linear_case(fl, 600, 1000, 1000, epilogue="RELU_AUX_BIAS", out_dtype="bf16", unfused=True, seed=4,
                       schedule="stream_k")
    assert got["info"]["stream_k_tiles"] > 0


def test_stream_k_repeated_executes_and_graph_replays(fl):
    """The stream-K flags reset themselves: the same plan executed back to back, then
    captured once in a CUDA graph and replayed, gives the oracle's result every time."""
    M, N, K = 600, 1000, 1000
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 23, bias_dtype="bf16")
    dA, dW, dB = inp["A"].cuda(), inp["W"].cuda(), inp["bias"].cuda()
    y, _, _, absdot = P.oracle_linear(A=inp["A"], W=inp["W"], bias=inp["bias"], epilogue="GELU_TANH_BIAS",
                                      out_dtype="bf16", M=M, N=N, K=K)
    plan = fl.Plan(M, N, K, kind="GELU_TANH_BIAS", out_dtype="bf16", lda=inp["A"].shape[1],
                   ldb=inp["W"].shape[1], schedule="stream_k")
    try:
        assert plan.info()["stream_k_tiles"] > 0
        outs = [P.poison((M, N), "bf16") for _ in range(3)]
        for o in outs:
            plan.execute(dA, dW, dB, out=o)
        assert plan.check() == fl.FL_OK, fl.fl_last_error()
        for i, o in enumerate(outs):
            P.check_close(P.to64(o), y, "bf16", absdot, f"execute {i}")
        og = P.poison((M, N), "bf16")
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            plan.execute(dA, dW, dB, out=og, stream=s)  # warm-up on the capture stream
            s.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                plan.execute(dA, dW, dB, out=og, stream=s)
        for r in range(3):
            og.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            P.check_close(P.to64(og), y, "bf16", absdot, f"graph replay {r}")
        assert plan.check() == fl.FL_OK, fl.fl_last_error()
        del g
    finally:
        plan.free()
