"""Register, spill and shared-memory figures of the built kernels (from `ptxas -v`).

build.py keeps the assembler's resource report beside the library.  The launch
configurations assume these figures, so a change that breaks one shows up here, on the
CPU, before it shows up as lost occupancy on the GPU:
- the fused kernel runs 320 threads a CTA, one CTA per SM: at most 204 registers;
- the dominant launch (ReLU + mask, bf16 out, CTA pair) spills only around its stream-K calls;
- the dReLU and bias-gradient kernels hold four 256-thread CTAs per SM (≤ 64 registers);
- the whole-vector LayerNorm holds six 128-thread CTAs per SM (≤ 85 registers) or four
  256-thread ones (≤ 64 registers).
Skipped when the report is missing (the library was not built here).
"""
from __future__ import annotations

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REPORT = os.path.join(ROOT, "gemm_bias_activation_tcgen05_b200", "ptxas_report.txt")


def _entries():
    if not os.path.exists(REPORT):
        pytest.skip("no ptxas report (library not built here)")
    out, cur = {}, None
    for line in open(REPORT):
        m = re.search(r"Compiling entry function '([^']+)'", line) or \
            re.search(r"Function properties for (\S+)", line)
        if m:
            cur = m.group(1)
            out.setdefault(cur, {})
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            out[cur]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out[cur]["regs"] = int(m.group(1))
    return out


def _select(entries, prefix):
    sel = {k: v for k, v in entries.items() if k.startswith(prefix)}
    assert sel, f"no kernel named {prefix}* in the report"
    return sel


def test_fused_kernel_fits_one_cta_of_320_threads():
    for name, v in _select(_entries(), "_ZN2fl19fl_gemm_epi_tcgen05").items():
        assert v["regs"] * 320 <= 65536, (name, v)


def test_dominant_launch_spills_only_around_its_stream_k_calls():
    # fl_gemm_epi_tcgen05<ACT_RELU, OUT_BF16, swap=false, tf32=false, pair=true>.  The two
    # stream-K steps (store a partial accumulator, add the others' partials) are out-of-line
    # calls, taken at most twice per CTA; the register saves around them are the only
    # spill traffic (the same kernel with empty callees spills as much; without the calls,
    # nothing).  The stream-K callees themselves do not spill.
    name = "_ZN2fl19fl_gemm_epi_tcgen05ILi1ELi1ELb0ELb0ELb1EEEv14CUtensorMap_stS1_S1_S1_NS_7KParamsE"
    e = _entries()
    assert name in e
    assert e[name]["spill"] <= 128, e[name]
    for callee in ("_ZN2fl16sk_store_partial", "_ZN2fl15sk_add_partials"):
        hits = {k: v for k, v in e.items() if k.startswith(callee)}
        assert all(v.get("spill", 0) == 0 for v in hits.values()), hits


@pytest.mark.parametrize("prefix,ctas,no_spill", [
    ("_ZN2fl23fl_relu_backward_kernel", 4, False),  # four CTAs of 256 threads per SM
    ("_ZN2fl19fl_bwd_bgrad_kernel", 3, True),       # three (its launch geometry assumes three)
])
def test_hbm_kernels_keep_their_ctas_of_256(prefix, ctas, no_spill):
    for name, v in _select(_entries(), prefix).items():
        assert v["regs"] * 256 * ctas <= 65536, (name, v)
        if no_spill:
            assert v["spill"] == 0, (name, v)


def test_vector_layernorm_keeps_its_ctas_per_sm():
    for name, v in _select(_entries(), "_ZN2fl23fl_layernorm_vec_kernel").items():
        threads, ctas = (128, 6) if "Li128EEEv" in name else (256, 4)
        assert v["regs"] * threads * ctas <= 65536, (name, v)
        assert v["spill"] == 0, (name, v)


def test_launchable_fused_kernels_do_not_spill():
    # Every instantiation of the fused kernel that a plan can launch keeps its epilogue in
    # registers: at most 16 bytes of spill stores and loads together (a register save or
    # two).  GeGLU with an fp32 output (act 4, out 2) is rejected by fl_plan and never
    # launched.  A change that
    # pushes one of these over the 168-register budget showed up as a slower whole-tile
    # schedule (tail_m2048 65.9 -> 70.9 us with 100 bytes of spills).
    e = _select(_entries(), "_ZN2fl19fl_gemm_epi_tcgen05")
    assert e
    bad = {k: v for k, v in e.items() if not k.startswith("_ZN2fl19fl_gemm_epi_tcgen05ILi4ELi2E") and v["spill"] > 16}
    assert not bad, bad
