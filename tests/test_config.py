"""The configuration choice of fl_plan, on the CPU through fl_plan_preview.

fl_plan_preview runs fl_plan's argument checks and configuration choice on the host
for a given SM count and shared-memory size, so these rules can be checked without a
GPU:
- M <= 128 takes the swap-AB layout (W on the 128-row side of the tensor core), except
  for GeGLU, an N-major B and fp32 operands;
- split-K over a cluster of S in {1, 2, 4} CTAs, with S <= the number of K blocks and
  tiles x S <= SMs;
- M > 128 takes CTA pairs (256-row tiles);
- every configuration fits the shared memory with at least two stages;
- the grid is persistent (at most one CTA per SM), a multiple of the cluster size.
"""
from __future__ import annotations

import random

import pytest

import gemm_bias_activation_tcgen05_b200 as fl

B200 = dict(num_sms=148, max_smem_per_block=232448)


def preview(M, N, K, dtype="bf16", **kw):
    compute = "32F_3XTF32" if dtype == "f32" else "32F"
    dev = {k: kw.pop(k) for k in ("num_sms", "max_smem_per_block") if k in kw}
    return fl.fl_plan_preview(M, N, K, dtype, compute, **{**B200, **dev}, **kw)


def bk_elems(dtype, info):
    # K elements of one pipeline stage: 128-byte swizzle atoms, two for 16-bit operands
    es = 4 if dtype == "f32" else 2
    atoms = 2 if dtype != "f32" else 1
    return atoms * 128 // es


def check_invariants(M, N, K, dtype, kind, info, num_sms=148, max_smem=232448):
    assert info["stages"] >= 2
    assert 0 < info["smem_bytes"] <= max_smem
    cluster = 2 if info["cta_pair"] else info["split_k"]
    assert info["grid"] % cluster == 0
    assert 0 < info["grid"] <= num_sms
    assert info["split_k"] in (1, 2, 4)
    num_kb = -(-K // bk_elems(dtype, info)) if K else 0
    if info["split_k"] > 1:
        assert info["swap_ab"] == 1
        assert info["split_k"] <= num_kb
        tiles = -(-N // 128) * -(-M // info["mma_n"])
        assert tiles * info["split_k"] <= num_sms
    if info["swap_ab"]:
        assert M <= 128 and kind != "GEGLU_TANH" and dtype != "f32"
        assert info["mma_n"] % 32 == 0 and info["mma_n"] >= M
        assert info["cta_pair"] == 0
    else:
        assert info["cta_pair"] == (1 if M > 128 else 0)
        assert info["tile_m"] == (256 if info["cta_pair"] else 128)
    if kind == "GEGLU_TANH":
        assert info["mma_n"] == 256 and info["tile_n"] == 128


@pytest.mark.parametrize("name,M,N,K,dtype,kw,expect", [
    # swap-AB with split-K for the HBM-bound small-M tails
    ("tail_m32", 32, 4096, 4096, "bf16", dict(kind="GELU_BIAS", out_dtype="f32", has_residual=True, scale=0.5),
     dict(swap_ab=1, split_k=4, mma_n=32, grid=128)),
    ("tail_m128", 128, 4096, 4096, "bf16", dict(kind="GELU_BIAS", out_dtype="f32", has_residual=True, scale=0.5),
     dict(swap_ab=1, split_k=4, mma_n=128, grid=128)),
    # CTA pairs beyond one 128-row tile
    ("tail_m512", 512, 4096, 4096, "bf16", dict(kind="GELU_BIAS", out_dtype="f32", has_residual=True, scale=0.5),
     dict(swap_ab=0, cta_pair=1, tile_m=256)),
    ("relu_aux_4096", 4096, 4096, 4096, "bf16", dict(kind="RELU_AUX_BIAS"),
     dict(swap_ab=0, cta_pair=1, tile_m=256, tile_n=256, grid=148)),
    # an N-major B keeps the normal layout even for M <= 128
    ("relu_bias_100x256x784", 100, 256, 784, "f16",
     dict(kind="RELU_BIAS", out_dtype="f32", bias_dtype="f32", bias_axis=1, b_major=1),
     dict(swap_ab=0, cta_pair=0, tile_m=128, grid=2)),
    # fp32 operands (3xTF32) on pairs
    ("linear_gelu_f32", 1024, 3072, 768, "f32", dict(kind="GELU_BIAS", out_dtype="f32", bias_dtype="f32"),
     dict(swap_ab=0, cta_pair=1)),
    # GeGLU: 256-wide UMMA over [gate; up], 128 output columns
    ("geglu", 8192, 3072, 768, "bf16", dict(kind="GEGLU_TANH"), dict(mma_n=256, tile_n=128, cta_pair=1)),
])
def test_configuration_of_the_workloads(name, M, N, K, dtype, kw, expect):
    info = preview(M, N, K, dtype, **kw)
    for k, v in expect.items():
        assert info[k] == v, (name, k, info)
    check_invariants(M, N, K, dtype, kw["kind"], info)


def test_invariants_over_random_shapes():
    rng = random.Random(7)
    kinds = ["NONE", "BIAS", "RELU_BIAS", "RELU_AUX_BIAS", "GELU_BIAS", "GELU_TANH_BIAS", "GEGLU_TANH",
             "GELU_AUX_BIAS", "GELU_SIGMOID_BIAS"]
    for _ in range(400):
        dtype = rng.choice(["bf16", "f16", "f32"])
        kind = rng.choice(kinds if dtype != "f32" else [k for k in kinds if k != "GEGLU_TANH"])
        out = "bf16" if kind == "GEGLU_TANH" else rng.choice(["bf16", "f16", "f32"])
        M = rng.choice([1, 7, 32, 33, 100, 128, 129, 255, 256, 511, 1000, 4096, 9000])
        # 16-byte row pitches: N a multiple of 8 (16-bit outputs), K a multiple of 8 (16-bit operands)
        N = 8 * rng.randint(1, 1200)
        K = rng.choice([0, 8, 64, 800, 784, 4096, 12288])
        sms = rng.choice([148, 132, 114, 16])
        smem = rng.choice([232448, 227 * 1024])
        info = preview(M, N, K, dtype, kind=kind, out_dtype=out, num_sms=sms, max_smem_per_block=smem)
        check_invariants(M, N, K, dtype, kind, info, sms, smem)


def test_unfused_twin_launch_count():
    assert preview(64, 256, 256, kind="RELU_BIAS", unfused=True)["launches_per_execute"] == 3
    assert preview(64, 256, 256, kind="GELU_BIAS", has_residual=True, scale=0.5,
                   unfused=True)["launches_per_execute"] == 5
    assert preview(64, 256, 256, kind="GEGLU_TANH", unfused=True)["launches_per_execute"] == 2
    assert preview(64, 256, 256, kind="NONE", unfused=True)["launches_per_execute"] == 1
    assert preview(64, 256, 256, kind="RELU_BIAS")["launches_per_execute"] == 1


def test_preview_applies_the_plan_checks():
    with pytest.raises(fl.FusedLinearError) as e:
        preview(64, 256, 256, kind="GELU_AUX_BIAS", unfused=True)
    assert e.value.status == fl.FL_ERR_UNSUPPORTED
    with pytest.raises(fl.FusedLinearError) as e:
        preview(0, 256, 256, kind="NONE")
    assert e.value.status == fl.FL_ERR_INVALID_ARG
    with pytest.raises(fl.FusedLinearError) as e:
        preview(64, 256, 256, kind="NONE", ldo=260)  # 520-byte rows: not a multiple of 16
    assert e.value.status == fl.FL_ERR_ALIGNMENT
    with pytest.raises(fl.FusedLinearError) as e:
        preview(64, 256, 256, kind="NONE", num_sms=1)
    assert e.value.status == fl.FL_ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K,kind,sk_tiles,sk_pairs", [
    (4096, 4096, 4096, "RELU_AUX_BIAS", 108, 74),  # 256 tiles: the last 34 plus one round of 74
    (512, 4096, 4096, "GELU_BIAS", 32, 64),        # 32 tiles, each split in two K halves
    (2048, 4096, 4096, "GELU_BIAS", 128, 74),      # 128 tiles: 54 plus one round, all of them
    (8192, 768, 3072, "NONE", 96, 74),             # GeGLU down projection
    (1024, 3072, 768, "GELU_TANH_BIAS", 0, 0),     # 48 tiles on 74 pairs: whole tiles
])
def test_stream_k_choice(M, N, K, kind, sk_tiles, sk_pairs):
    # the default schedule keeps whole tiles; stream-K, when asked for, splits as described
    auto = preview(M, N, K, kind=kind, out_dtype="bf16")
    assert auto["stream_k_tiles"] == 0 and auto["stream_k_pairs"] == 0
    info = preview(M, N, K, kind=kind, out_dtype="bf16", schedule="stream_k")
    check_invariants(M, N, K, "bf16", kind, info)
    T = -(-M // 256) * -(-N // info["tile_n"])
    assert info["stream_k_tiles"] == sk_tiles
    assert info["stream_k_pairs"] == sk_pairs
    if sk_tiles:
        # every stream-K range spans at least one whole tile, or (fewer tiles than half the
        # pairs) each tile is split in exactly two K halves
        units = sk_tiles * -(-K // 128)
        assert units // sk_pairs >= -(-K // 128) or sk_pairs == 2 * sk_tiles
        # the tiles before the stream-K ones are whole rounds of the 74 pairs
        assert (T - sk_tiles) % 74 == 0
        assert info["grid"] == 2 * max(sk_pairs, 74 if T > sk_tiles else 0)


@pytest.mark.parametrize("M,N,K,kind,sk_tiles", [
    (1024, 3072, 768, "GELU_TANH_BIAS", 0),    # 48 tiles: more than half the pairs, fewer than all
    (8192, 3072, 768, "GEGLU_TANH", 102),      # 28 left over plus one round
    (8192, 8192, 1024, "BIAS", 136),
    (600, 1000, 1000, "GELU_BIAS", 12),
])
def test_stream_k_forced(M, N, K, kind, sk_tiles):
    info = preview(M, N, K, kind=kind, out_dtype="bf16", schedule="stream_k")
    check_invariants(M, N, K, "bf16", kind, info)
    assert info["stream_k_tiles"] == sk_tiles
    dp = preview(4096, 4096, 4096, kind="RELU_AUX_BIAS", out_dtype="bf16", schedule="data_parallel")
    assert dp["stream_k_tiles"] == 0 and dp["grid"] == 148


def test_stream_k_only_for_16_bit_pairs():
    for kw in [dict(M=100, N=4096, K=4096), dict(M=128, N=4096, K=4096)]:   # swap-AB
        assert preview(kw["M"], kw["N"], kw["K"], kind="GELU_BIAS", out_dtype="f32",
                       schedule="stream_k")["stream_k_tiles"] == 0
    assert preview(1024, 3072, 768, "f32", kind="GELU_BIAS", out_dtype="f32",
                   schedule="stream_k")["stream_k_tiles"] == 0
    # a full last round stays data-parallel
    assert preview(256 * 74, 256, 1024, kind="BIAS", out_dtype="bf16", schedule="stream_k")["stream_k_tiles"] == 0


def test_unknown_schedule_is_rejected():
    with pytest.raises(fl.FusedLinearError):
        e = fl.make_epilogue(kind="BIAS")
        e.schedule = 7
        info = fl.fl_plan_info()
        st = fl.LIB.fl_plan_preview(512, 512, 512, fl.FL_BF16, fl.FL_COMPUTE_32F, fl.ctypes.byref(e), 148, 232448,
                                    fl.ctypes.byref(info))
        fl._check(st, "preview")
