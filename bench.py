"""Benchmark of the B200 fused linear layer.

One step = one pass of the whole hot path over one batch of synthetic input:
every synthetic workload of the fused linear layer once, each through the C ABI
as a single fused launch —
  relu_bias_100x256x784                relu(W·x + b), fp16, B stored [K,N], bias per row
  linear_gelu_f32_1024x3072x768        exact GELU, fp32 operands (3xTF32 on the tensor cores)
  linear_gelu_tanh_bf16_1024x3072x768  tanh GELU, bf16
  geglu_mlp_8192x3072x768              dual gate/up GEMM with gelu_tanh(g)·u, then down_proj
  relu_aux_4096                        RELU_AUX_BIAS forward + dReLU backward
  tail_m{32,128,512,2048}              bias → GELU(erf) → +residual → ×0.5, fp32 out
The headline value is the whole step's algorithmic TFLOP/s (2·M·N·K per GEMM);
each launch is also timed with CUDA events on its stream for the per-workload
breakdown and the roofline of the dominant kernel.

Every workload owns its tensors, so a kernel's operands were last touched one
full step (several hundred MB of other traffic) earlier: the inputs of a step
are larger than L2 and nothing is L2-resident between iterations.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun): independent replicas, weak scaling, max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused Linear+bias+act TFLOP/s (% of BF16 tensor peak); GeGLU MLP fwd µs"
SUITE = ["relu_bias_100x256x784", "linear_gelu_f32_1024x3072x768", "linear_gelu_tanh_bf16_1024x3072x768",
         "geglu_mlp_8192x3072x768", "relu_aux_4096", "tail_m32", "tail_m128", "tail_m512", "tail_m2048"]
DOMINANT = "relu_aux_4096"   # the largest single fused launch of the step


def workload_desc(names):
    """The `config.workload` string of both arms: the step's workloads by name and size."""
    return "all synthetic workloads of the fused linear layer, one fused launch each: " + ", ".join(names)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of a captured graph")
    ap.add_argument("--profile", default=None, metavar="WORKLOAD",
                    help="run only this workload's launches (warm-up + steps), print nothing; for ncu captures")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    """The largest of the ranks' values (each rank's device time): the job ends with its
    slowest replica.  A one-element all-reduce, on the GPU under NCCL, on the host under gloo."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(ws, flops_per_step, steps, total_ms):
    """Whole-job throughput of N replicas (weak scaling): every rank runs `steps` steps of
    `flops_per_step`, and the job takes the slowest rank's `total_ms`."""
    return ws * flops_per_step * steps / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks
REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))


class ClockSampler:
    """SM clock and clock-event reasons, sampled while the context is open.

    NVML is read every 5 ms from a host thread (read-only queries); without NVML,
    nvidia-smi prints a sample every 200 ms.  Samples are (time.time(), sm MHz, max MHz,
    reasons).  phase(name) opens a named interval that lasts until the next phase() or
    the end, so that the summary of an interval holds the samples taken while that
    work ran: the timed region is preceded by a warm pass of at least one second,
    which guarantees samples under the same load at any number of steps."""
    PERIOD_S = 0.005

    def __init__(self, gpu_index, pci_bus_id=None):
        self.idx = gpu_index
        self.pci = pci_bus_id
        self.proc = None
        self.thread = None
        self.samples = []
        self.lines = []
        self.phases = []  # (name, t_start)
        self.source = None
        self._stop = False

    def phase(self, name):
        self.phases.append((name, time.time()))

    def _nvml_loop(self, nv, h):
        while not self._stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), float(sm), float(mx),
                                     frozenset(n for n, b in REASON_BITS if rs & b)))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = None
            if self.pci:
                try:
                    h = nv.nvmlDeviceGetHandleByPciBusId(self.pci)
                except Exception:
                    h = None
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            self.source = "nvml, 5 ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={SMI_QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi, 200 ms"
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        self._stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def _all(self):
        """NVML samples, or the nvidia-smi lines parsed into the same form."""
        import datetime
        out = list(self.samples)
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(f[2]), float(f[3])
            except ValueError:
                continue
            rs = frozenset(n for (n, _), v in zip(REASON_BITS, f[6:10]) if v.lower().startswith("active"))
            out.append((ts, sm, mx, rs))
        return sorted(out, key=lambda x: x[0])

    def summary(self, name=None):
        """Median SM clock, max clock and every reason seen, over the samples of phase
        `name` (all phases when None)."""
        smp = self._all()
        if name is not None:
            bounds = [(n, t, self.phases[i + 1][1] if i + 1 < len(self.phases) else float("inf"))
                      for i, (n, t) in enumerate(self.phases)]
            sel = [(t0, t1) for n, t0, t1 in bounds if n == name]
            smp = [x for x in smp if any(t0 <= x[0] < t1 for t0, t1 in sel)]
        elif self.phases:
            smp = [x for x in smp if x[0] >= self.phases[0][1]]
        mx = max((x[2] for x in smp), default=None)
        reasons = sorted(set().union(*[x[3] for x in smp])) if smp else []
        if not smp:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": reasons, "samples": 0, "source": self.source}
        return {"sm_mhz": statistics.median(x[1] for x in smp), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(smp), "source": self.source}


SMI_QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# ---------------------------------------------------------------- our arm
class Suite:
    """Device tensors and plans of every workload; launch() runs one step."""

    def __init__(self, fl, seed=0):
        import torch
        import workloads
        self.fl, self.torch = fl, torch
        self.items = []
        self.flops = 0.0
        self.min_bytes = {}
        for name in SUITE:
            w = workloads.get(name)
            if w.dtype == "f32" and not self._f32_supported():
                continue
            inp = workloads.make_inputs(w, seed)
            it = {"w": w, "host": inp}
            if w.kind == "geglu":
                x, Wgu, Wd = inp["x"], torch.cat([inp["Wg"], inp["Wu"]], 0), inp["Wd"]
                it["dev"] = {"x": x.cuda(), "Wgu": Wgu.cuda(), "Wd": Wd.cuda()}
                it["h"] = torch.empty(w.M, w.N, dtype=torch.bfloat16, device="cuda")
                it["y"] = torch.empty(w.M, w.K, dtype=torch.bfloat16, device="cuda")
                it["plans"] = [fl.Plan(w.M, w.N, w.K, kind="GEGLU_TANH", out_dtype="bf16"),
                               fl.Plan(w.M, w.K, w.N, kind="NONE", out_dtype="bf16")]
                it["host_in"] = {"x": x, "Wgu": Wgu, "Wd": Wd}
                it["outs"] = ["y"]
                self.min_bytes[name] = 2 * (w.M * w.K + 2 * w.N * w.K + 2 * w.M * w.N + w.K * w.N + w.M * w.K)
            else:
                td = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
                dev = {k: v.cuda() for k, v in inp.items()}
                it["dev"] = dev
                it["out"] = torch.empty(w.M, w.N, dtype=td[w.out_dtype], device="cuda")
                it["aux"] = (torch.empty(w.M, (w.N + 31) // 32, dtype=torch.int32, device="cuda")
                             if w.epilogue == "RELU_AUX_BIAS" else None)
                it["dpre"] = (torch.empty(w.M, w.N, dtype=torch.bfloat16, device="cuda")
                              if w.kind == "relu_aux" else None)
                it["plans"] = [fl.Plan(w.M, w.N, w.K, dtype=w.dtype,
                                       compute="32F_3XTF32" if w.dtype == "f32" else "32F",
                                       kind=w.epilogue, out_dtype=w.out_dtype, bias_dtype=w.bias_dtype or "bf16",
                                       residual_dtype=w.dtype, bias_axis=w.bias_axis, has_residual=w.residual,
                                       scale=w.scale, b_major=w.b_major)]
                it["host_in"] = {k: v for k, v in inp.items() if k != "grad" or w.kind == "relu_aux"}
                it["outs"] = ["out"] + (["aux"] if it["aux"] is not None else []) + \
                             (["dpre"] if it["dpre"] is not None else [])
                es = {"f16": 2, "bf16": 2, "f32": 4}
                b = es[w.dtype] * (w.M * w.K + w.N * w.K) + es[w.out_dtype] * w.M * w.N
                if w.bias_dtype:
                    b += es[w.bias_dtype] * (w.M if w.bias_axis else w.N)
                if w.residual:
                    b += es[w.dtype] * w.M * w.N
                if it["aux"] is not None:
                    b += 4 * w.M * ((w.N + 31) // 32)
                self.min_bytes[name] = b
            self.flops += w.flops
            self.items.append(it)

    @staticmethod
    def _f32_supported():
        return True

    def launches_per_step(self):
        n = 0
        for it in self.items:
            n += len(it["plans"]) + (1 if it.get("dpre") is not None else 0)
        return n

    def run_item(self, it, stream):
        fl, w, d = self.fl, it["w"], it["dev"]
        if w.kind == "geglu":
            it["plans"][0].execute(d["x"], d["Wgu"], out=it["h"], stream=stream)
            it["plans"][1].execute(it["h"], d["Wd"], out=it["y"], stream=stream)
            return
        W = d["B"] if w.b_major else d["W"]
        it["plans"][0].execute(d["A"], W, d.get("bias"), it["aux"], d.get("residual"), it["out"], stream=stream)
        if it["dpre"] is not None:
            fl.fl_relu_backward(d["grad"], it["aux"], it["dpre"], w.M, w.N, "bf16", stream=stream)

    def check(self):
        for it in self.items:
            for p in it["plans"]:
                st = p.check()
                if st != self.fl.FL_OK:
                    raise RuntimeError(f"{it['w'].name}: status {st}: {self.fl.fl_last_error()}")


def run_ours(args):
    import torch
    import gemm_bias_activation_tcgen05_b200 as fl

    ws, rank, local = dist_setup(args.gpus)
    pk = peaks()
    suite = Suite(fl, seed=rank)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    # ---- warm-up (untimed), then a correctness status check of every plan
    for _ in range(max(args.warmup, 3)):
        for it in suite.items:
            suite.run_item(it, sh)
    torch.cuda.synchronize()
    suite.check()

    # ---- timed region: K steps captured once as a CUDA graph, so the replay has no
    # host enqueue gaps between launches; the kernels are launched with programmatic
    # dependent launch, so a kernel's prologue overlaps its predecessor's tail.
    # Per-workload times come from a second graph with an event pair around every
    # workload (an event node between two kernels serialises them fully).
    n_items = len(suite.items)
    use_graph = not args.no_graph
    n_ev = min(args.steps, 20)  # steps of the per-workload breakdown graph
    ev = [[(torch.cuda.Event(enable_timing=True, external=use_graph),
            torch.cuda.Event(enable_timing=True, external=use_graph)) for _ in range(n_items)]
          for _ in range(n_ev)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def k_steps(stream_handle, with_events):
        for s in range(n_ev if with_events else args.steps):
            for i, it in enumerate(suite.items):
                if with_events:
                    ev[s][i][0].record()
                suite.run_item(it, stream_handle)
                if with_events:
                    ev[s][i][1].record()

    graph = ev_graph = None
    if use_graph:
        graph, ev_graph = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            k_steps(torch.cuda.current_stream().cuda_stream, False)
        with torch.cuda.graph(ev_graph):
            k_steps(torch.cuda.current_stream().cuda_stream, True)
        graph.replay()  # one untimed replay of the captured steps
        torch.cuda.synchronize()
    pci = None
    try:
        pr = torch.cuda.get_device_properties(torch.cuda.current_device())
        pci = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:
        pass
    clk = ClockSampler(local, pci).__enter__()
    # warm pass: replays of the K steps for at least one second, so that the clocks and
    # the power draw settle under the step's load and the sampler has samples of it at
    # any K; then the timed region, bracketed by a barrier and a synchronize
    clk.phase("warm")
    t_warm = time.time()
    while True:
        if graph is not None:
            graph.replay()
        else:
            k_steps(sh, False)
        torch.cuda.synchronize()
        if time.time() - t_warm >= 1.0:
            break
    barrier(ws)
    torch.cuda.synchronize()
    clk.phase("timed")
    t0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        k_steps(sh, False)
    t1.record(stream)
    torch.cuda.synchronize()
    clk.phase("after")
    barrier(ws)
    total_ms = max_over_ranks(t0.elapsed_time(t1), ws)
    suite.check()
    ms_step = total_ms / args.steps
    # per-workload breakdown (outside the timed region)
    if ev_graph is not None:
        ev_graph.replay()
    else:
        k_steps(sh, True)
    torch.cuda.synchronize()
    per_item = {}
    for i, it in enumerate(suite.items):
        times = [ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(n_ev)]
        per_item[it["w"].name] = {"ms_mean": sum(times) / len(times), "ms_median": statistics.median(times)}

    # ---- e2e through the public API with host buffers: pinned H2D of every operand,
    # the launches, D2H of every result, all inside the timed region
    e2e = e2e_measure(suite, stream, sh, args, ws)

    value = job_tflops(ws, suite.flops, args.steps, total_ms)
    breakdown = {}
    for it in suite.items:
        w = it["w"]
        t = per_item[w.name]["ms_mean"]
        tfl = w.flops / (t * 1e-3) / 1e12
        gbs = suite.min_bytes[w.name] / (t * 1e-3) / 1e9
        roof_t = max(w.flops / (pk["bf16_tflops"] * 1e12), suite.min_bytes[w.name] / (pk["hbm_gbs"] * 1e9))
        breakdown[w.name] = {"us": round(t * 1e3, 2), "tflops": round(tfl, 1), "gbs_min_bytes": round(gbs, 1),
                             "roofline_us": round(roof_t * 1e6, 2), "roofline_frac": round(roof_t / (t * 1e-3), 3)}
    # each workload's launches alone, as the time they add to a stream (L2 flushed before each)
    flush_b = L2Flush()
    for it in suite.items:
        fn = lambda it=it: suite.run_item(it, torch.cuda.current_stream().cuda_stream)  # noqa: E731
        breakdown[it["w"].name]["us_in_stream"] = round(time_in_stream(fn, 20, flush_b) * 1e3, 2)
    del flush_b
    dom = suite.items[[it["w"].name for it in suite.items].index(DOMINANT)]
    dom_w = dom["w"]
    # the dominant fused GEMM launch alone (its dReLU follows inside the same event pair,
    # so the forward is timed separately below on the same stream), each launch after an
    # L2 flush: a burst of isolated launches, compared with the burst bf16 peak
    clk.phase("roofline")
    fwd_ms, fwd_ms_stream = time_single_launch(suite, dom, stream, sh, reps=max(10, min(100, args.steps // 2)))
    clk.phase("after")
    clk.phase("side")
    hbm = time_backward(fl, pk)
    sig = time_gelu_sigmoid(fl, pk)
    fusion = time_fusion(suite, fl)
    clk.__exit__(None, None, None)
    achieved = dom_w.flops / (fwd_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    roof_clk = clk.summary("roofline")
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 3), "traffic": profiled_traffic(), "kernel": "fl_gemm_epi_tcgen05",
                "launch": f"{DOMINANT} forward (M=N=K=4096, RELU_AUX_BIAS)", "us": round(fwd_ms * 1e3, 2),
                "peak_kind": f"{pk['src']} bf16 burst (the launch is timed alone, after an L2 flush each time)",
                "frac_of_sustained": round(achieved / pk["bf16_tflops_sustained"], 3),
                "us_in_stream": round(fwd_ms_stream * 1e3, 2),
                "frac_in_stream": round(dom_w.flops / (fwd_ms_stream * 1e-3) / 1e12 / peak, 3),
                "sm_mhz": roof_clk["sm_mhz"],
                "us_x_ghz": (round(fwd_ms * 1e3 * roof_clk["sm_mhz"] / 1e3, 2) if roof_clk["sm_mhz"] else None)}
    timed_clk = clk.summary("timed")
    warm_clk = clk.summary("warm")
    use = timed_clk if timed_clk["samples"] else warm_clk
    clocks = {"sm_mhz": use["sm_mhz"], "sm_max_mhz": use["sm_max_mhz"] or warm_clk["sm_max_mhz"],
              "reasons": sorted(set(timed_clk["reasons"]) | set(warm_clk["reasons"])),
              "samples_timed": timed_clk["samples"], "samples_warm": warm_clk["samples"],
              "sm_mhz_warm": warm_clk["sm_mhz"], "source": clk.source,
              "window": "timed region, and the >= 1 s warm pass of the same replays just before it"}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc([it["w"].name for it in suite.items]),
                   "timed_as": "one CUDA graph of the K steps" if use_graph else "eager launches",
                   "flops_per_step": suite.flops, "parallelism": f"replicas x{ws}",
                   "l2": "inputs larger than L2: every workload owns its operands; a step touches "
                         f"{sum(suite.min_bytes.values()) / 1e6:.0f} MB"},
        "impl": "ours",
        "geglu_mlp_fwd_us": breakdown.get("geglu_mlp_8192x3072x768", {}).get("us"),
        "pct_of_bf16_peak": round(100 * value / ws / pk["bf16_tflops"], 1),
        "e2e": e2e,
        "gpu_launches": suite.launches_per_step() * args.steps,
        "roofline": roofline,
        "clocks": clocks,
        "breakdown": breakdown,
        "hbm_kernels": hbm,
        "gelu_sigmoid_1024x3072x768_bf16": sig,
        "fusion": fusion,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, ev_graph
    torch.cuda.synchronize()
    for it in suite.items:
        for p in it["plans"]:
            p.free()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


class L2Flush:
    """Flush L2 between timed launches: write a 256 MB buffer (larger than the 126 MB L2),
    then read another 256 MB buffer, so that the written lines are back in DRAM before the
    timed launch and it does not pay for their write-back.  Runs outside the event pair."""

    def __init__(self):
        import torch
        n = 256 * 1024 * 1024 // 4
        self.w = torch.empty(n, dtype=torch.int32, device="cuda")
        self.r = torch.zeros(n, dtype=torch.float32, device="cuda")  # fp32: sum() reads it without a cast copy

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def time_in_graph(fn, reps, flush=None):
    """Mean CUDA-event time (ms) of fn(), each launch preceded by an L2 flush (outside the
    event pair).  The whole sequence (flush, event, fn, event) x reps is captured once as a
    CUDA graph and replayed, so the GPU never waits for the host inside an event pair (timed
    one launch at a time from Python, a short kernel's events would also hold the host's
    enqueue latency).  fn must launch on the current stream."""
    import torch
    fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(reps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for a, b in evs:
            if flush is not None:
                flush()
            a.record()
            fn()
            b.record()
    g.replay()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / reps
    del g
    return ms


def time_single_launch(suite, it, stream, sh, reps):
    """The workload's first launch alone, each after an L2 flush: (event pair around each
    launch, in-stream difference) in ms."""
    d = it["dev"]
    flush = L2Flush()
    fn = lambda: it["plans"][0].execute(d["A"], d["W"], d.get("bias"), it["aux"], d.get("residual"),  # noqa: E731
                                         it["out"], stream=None)
    ms = time_in_graph(fn, reps, flush)
    ms_stream = time_in_stream(fn, 20, flush)
    del flush
    return ms, ms_stream


def hbm_runs(fl, sh):
    """The HBM-bound kernels beside the fused layer, on resident synthetic inputs: the
    backward with and without the fused bias gradient on the relu_aux_4096 shape
    (4096 x 4096 bf16) and the LayerNorm of the tail_m2048 output.  Returns
    {name: (launch, algorithmic bytes)}."""
    import torch
    M = N = 4096
    g = torch.Generator(device="cpu").manual_seed(5)
    grad = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    v = (torch.randn(M, N, generator=g) * 3).to(torch.bfloat16).cuda()
    mask = torch.randint(-2 ** 31, 2 ** 31 - 1, (M, N // 32), generator=g, dtype=torch.int32).cuda()
    dpre = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dbias = torch.empty(N, dtype=torch.float32, device="cuda")
    nbytes = fl.fl_bias_grad_workspace_size(M, N, "bf16")
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    runs = {
        "drelu_bgrad_4096x4096_bf16": (lambda: fl.fl_drelu_bgrad(grad, mask, dpre, dbias, M, N, "bf16", ws, nbytes,
                                                                 stream=sh),
                                       2 * M * N * 2 + M * N // 8 + 4 * N),
        "dgelu_bgrad_4096x4096_bf16": (lambda: fl.fl_dgelu_bgrad(grad, v, dpre, dbias, M, N, "bf16", ws, nbytes,
                                                                 stream=sh),
                                       3 * M * N * 2 + 4 * N),
        # the same dReLU without the bias gradient, and the plain dReLU kernel of the bench step
        "drelu_4096x4096_bf16": (lambda: fl.fl_drelu_bgrad(grad, mask, dpre, None, M, N, "bf16", stream=sh),
                                 2 * M * N * 2 + M * N // 8),
        "relu_backward_4096x4096_bf16": (lambda: fl.fl_relu_backward(grad, mask, dpre, M, N, "bf16", stream=sh),
                                         2 * M * N * 2 + M * N // 8),
    }
    # LayerNorm of the BERT-tail output rows (tail_m2048: [2048, 4096] fp32 -> bf16)
    Ml, Nl = 2048, 4096
    y = torch.randn(Ml, Nl, generator=g).cuda()
    gam = torch.ones(Nl, device="cuda")
    bet = torch.zeros(Nl, device="cuda")
    zl = torch.empty(Ml, Nl, dtype=torch.bfloat16, device="cuda")
    runs["layernorm_2048x4096_f32_to_bf16"] = (
        lambda: fl.fl_layernorm(y, gam, bet, zl, Ml, Nl, "f32", "bf16", "f32", eps=1e-12, stream=sh),
        Ml * Nl * (4 + 2) + 2 * 4 * Nl)
    return runs


HBM_KERNELS = ("drelu_bgrad_4096x4096_bf16", "dgelu_bgrad_4096x4096_bf16", "drelu_4096x4096_bf16",
               "relu_backward_4096x4096_bf16", "layernorm_2048x4096_f32_to_bf16")


def time_in_stream(fn, reps, flush):
    """Mean time (ms) that one launch of fn() adds to a stream, each launch after an L2
    flush: a CUDA graph of reps x (flush, fn) minus a graph of reps x flush, each replay
    bracketed by one event pair (median of five replays).  An event pair around every
    launch (time_in_graph) also holds the event records' own cost, about 4.5 us for an
    isolated launch on this GPU; this difference does not, and still holds the launch's
    start-up and drain in the stream.  fn must launch on the current stream."""
    import statistics
    import torch

    def graph_ms(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                body()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        del g
        return statistics.median(ts)

    def both():
        flush()
        fn()

    fn()
    torch.cuda.synchronize()
    return (graph_ms(both) - graph_ms(flush)) / reps


def time_backward(fl, pk, reps=20):
    """Each HBM-bound kernel of hbm_runs() after a 256 MB L2 flush: the time it adds to
    the stream (time_in_stream), achieved GB/s of the algorithmic bytes from it, and the
    fraction of the measured HBM copy bandwidth; us_event_pair is the same launch inside
    its own event pair (time_in_graph), for comparison."""
    import torch
    runs = hbm_runs(fl, None)
    flush = L2Flush()
    out = {}
    for name, (fn, algo_bytes) in runs.items():
        ms_ev = time_in_graph(fn, reps, flush)
        ms = time_in_stream(fn, reps, flush)
        gbs = algo_bytes / (ms * 1e-3) / 1e9
        out[name] = {"us": round(ms * 1e3, 2), "us_event_pair": round(ms_ev * 1e3, 2), "algorithmic_bytes": algo_bytes,
                     "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 3),
                     "timed_as": "in-stream: graph of (L2 flush, launch) x 20 minus graph of flush x 20"}
    del flush
    return out


def time_gelu_sigmoid(fl, pk, reps=10):
    """The GELU_SIGMOID_BIAS epilogue on the [gelu] unit-test shape (x [1024,768],
    W [3072,768], bf16 out), each launch after a 256 MB L2 flush."""
    import torch
    import workloads
    M, N, K = 1024, 3072, 768
    inp = workloads.ragged_linear_inputs(M, N, K, "bf16", 3, bias_dtype="bf16", pad=1)
    A, W, b = inp["A"].cuda(), inp["W"].cuda(), inp["bias"].cuda()
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    plan = fl.Plan(M, N, K, kind="GELU_SIGMOID_BIAS", out_dtype="bf16")
    flush = L2Flush()
    try:
        ms = time_in_graph(lambda: plan.execute(A, W, b, out=out), reps, flush)
        assert plan.check() == fl.FL_OK
    finally:
        plan.free()
    tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    return {"us": round(ms * 1e3, 2), "tflops": round(tf, 1), "frac_of_bf16_burst": round(tf / pk["bf16_tflops"], 3)}


FUSION_SET = ["linear_gelu_tanh_bf16_1024x3072x768", "geglu_mlp_8192x3072x768", "relu_aux_4096", "tail_m2048"]


def _time_launch(fn, flush, reps):
    """Mean CUDA-event time (ms) of fn(), each launch after an L2 flush (time_in_graph)."""
    return time_in_graph(fn, reps, flush)


def time_fusion(suite, fl, reps=10):
    """What fusion buys, per workload: the fused launch, the bare GEMM (epilogue NONE,
    same operands and output type) and the unfused twin (the bare GEMM into an
    intermediate, then one elementwise kernel per epilogue step), each after an L2
    flush.  epilogue_overhead = fused / bare − 1; round_trip_us = unfused − fused.
    For GeGLU the dual gate/up GEMM is compared (the down projection is the same plain
    GEMM either way).  A workload whose measurement fails records the error instead."""
    import torch
    flush = L2Flush()
    sh = None  # the current stream at launch time (the capture stream inside a graph)
    out = {}
    for it in suite.items:
        w = it["w"]
        if w.name not in FUSION_SET:
            continue
        plans = []
        try:
            d = it["dev"]
            if w.kind == "geglu":
                h2 = torch.empty(w.M, 2 * w.N, dtype=torch.bfloat16, device="cuda")
                bare = fl.Plan(w.M, 2 * w.N, w.K, kind="NONE", out_dtype="bf16")
                unf = fl.Plan(w.M, w.N, w.K, kind="GEGLU_TANH", out_dtype="bf16", unfused=True)
                plans += [bare, unf]
                fused_fn = lambda: it["plans"][0].execute(d["x"], d["Wgu"], out=it["h"], stream=sh)
                bare_fn = lambda: bare.execute(d["x"], d["Wgu"], out=h2, stream=sh)
                unf_fn = lambda: unf.execute(d["x"], d["Wgu"], out=it["h"], stream=sh)
            else:
                compute = "32F_3XTF32" if w.dtype == "f32" else "32F"
                Wt = d["B"] if w.b_major else d["W"]
                ob = torch.empty_like(it["out"])
                bare = fl.Plan(w.M, w.N, w.K, dtype=w.dtype, compute=compute, kind="NONE", out_dtype=w.out_dtype,
                               b_major=w.b_major)
                unf = fl.Plan(w.M, w.N, w.K, dtype=w.dtype, compute=compute, kind=w.epilogue, out_dtype=w.out_dtype,
                              bias_dtype=w.bias_dtype or "bf16", residual_dtype=w.dtype, bias_axis=w.bias_axis,
                              has_residual=w.residual, scale=w.scale, b_major=w.b_major, unfused=True)
                plans += [bare, unf]
                args = (d["A"], Wt, d.get("bias"), it["aux"], d.get("residual"))
                fused_fn = lambda: it["plans"][0].execute(*args, it["out"], stream=sh)
                bare_fn = lambda: bare.execute(d["A"], Wt, out=ob, stream=sh)
                unf_fn = lambda: unf.execute(*args, ob, stream=sh)
            t_f = _time_launch(fused_fn, flush, reps)
            t_b = _time_launch(bare_fn, flush, reps)
            t_u = _time_launch(unf_fn, flush, reps)
            for p in plans + [it["plans"][0]]:
                if p.check() != fl.FL_OK:
                    raise RuntimeError(fl.fl_last_error())
            out[w.name] = {"fused_us": round(t_f * 1e3, 2), "bare_gemm_us": round(t_b * 1e3, 2),
                           "unfused_us": round(t_u * 1e3, 2), "unfused_launches": unf.info()["launches_per_execute"],
                           "epilogue_overhead": round(t_f / t_b - 1.0, 3), "round_trip_us": round((t_u - t_f) * 1e3, 2)}
        except Exception as e:  # keep the rest of the line
            out[w.name] = {"error": str(e)[:200]}
        finally:
            try:
                torch.cuda.synchronize()
                for p in plans:
                    p.free()
            except Exception:
                pass
    del flush
    return out


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "fl_gemm_epi_relu_aux_4096.json")


def kernel_source_hash():
    """First 16 hex digits of the SHA-256 of the fused kernel's source files."""
    h = hashlib.sha256()
    for f in ("fl_gemm.cuh", "fl_ptx.cuh"):
        h.update(open(os.path.join(ROOT, "gemm_bias_activation_tcgen05_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes (read + write) per launch of the dominant kernel from the committed ncu
    record (profiles/fl_gemm_epi_relu_aux_4096.json), or None when the kernel source has
    changed since the counters were taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    try:
        d = json.load(open(TRAFFIC_FILE))
        if d.get("kernel_source_sha256_16") != kernel_source_hash():
            return None
        return float(d["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError, TypeError):
        return None


def e2e_measure(suite, stream, sh, args, ws):
    import torch
    host = []
    h2d = d2h = 0
    for it in suite.items:
        pin_in = {k: v.pin_memory() for k, v in it["host_in"].items()}
        outs = {}
        for k in it["outs"]:
            t = it[k] if k in it else None
            if t is None:
                continue
            outs[k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        host.append((it, pin_in, outs))
        h2d += sum(v.numel() * v.element_size() for v in pin_in.values())
        d2h += sum(v.numel() * v.element_size() for v in outs.values())

    # Three streams: host->device copies, the launches, device->host copies.  Workload
    # i+1's inputs travel while workload i computes and workload i-1's results travel
    # back (the two copy directions use separate engines).  Events order every reuse of
    # a device buffer across steps: a workload's inputs are overwritten only after its
    # previous launches finished, and its outputs only after their previous read-back.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(host)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    started = [False] * n

    def step():
        for i, (it, pin_in, outs) in enumerate(host):
            with torch.cuda.stream(s_in):
                if started[i]:
                    s_in.wait_event(ev_done[i])
                for k, v in pin_in.items():
                    it["dev"][k].copy_(v, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if started[i]:
                stream.wait_event(ev_out[i])
            suite.run_item(it, sh)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                for k, v in outs.items():
                    v.copy_(it[k], non_blocking=True)
                ev_out[i].record(s_out)
            started[i] = True

    steps = max(3, min(args.steps, 10))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        step()
    b.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), ws) / steps
    return {"value": round(ws * suite.flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3)}


# ---------------------------------------------------------------- oracle on the host cores
_ORACLE_INPUTS = {}


def _oracle_sample(seconds, rows_per_chunk=64, chunks=None):
    """Run the oracle (as it stands) over row-slices of every workload until about
    `seconds` of CPU work is done (or exactly `chunks` chunks of rows);
    returns (flops, elapsed, cores, description)."""
    import numpy as np
    import oracle
    import workloads
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    flops, elapsed, parts = 0.0, 0.0, []
    names = [n for n in SUITE]
    data = _ORACLE_INPUTS  # generated once per process, outside the timed CPU work
    for n in names:
        if n not in data:
            w = workloads.get(n)
            data[n] = (w, {k: v.double().numpy() for k, v in workloads.make_inputs(w, 0).items()})
    r0 = 0
    done = 0
    while (elapsed < seconds if chunks is None else done < chunks) and r0 < 8192:
        done += 1
        for n in names:
            w, inp = data[n]
            if r0 >= w.M:
                continue
            r1 = min(w.M, r0 + rows_per_chunk)
            t = time.perf_counter()
            if w.kind == "geglu":
                oracle.geglu_mlp(inp["x"][r0:r1], inp["Wg"], inp["Wu"], inp["Wd"], "bf16")
                f = 2.0 * (r1 - r0) * w.K * 3 * w.N
            else:
                Wm = inp["B"] if w.b_major else inp["W"]
                bias = inp.get("bias")
                if bias is not None and w.bias_axis == 1:
                    bias = bias[r0:r1]
                res = inp.get("residual")
                y, aux, v = oracle.fused_linear(inp["A"][r0:r1], Wm, bias, epilogue=w.epilogue,
                                                out_dtype=w.out_dtype, bias_axis=w.bias_axis, b_major=w.b_major,
                                                residual=None if res is None else res[r0:r1], scale=w.scale)
                if aux is not None:
                    oracle.drelu(inp["grad"][r0:r1], aux, w.N, "bf16")
                f = 2.0 * (r1 - r0) * w.N * w.K
            elapsed += time.perf_counter() - t
            flops += f
        r0 += rows_per_chunk
    desc = (f"oracle (numpy/scipy fp64) on row slices [0:{r0}) of every workload "
            f"({flops / 1e9:.1f} GFLOP, {elapsed:.1f} s)")
    return flops, elapsed, cores, desc


def _oracle_pass(rows):
    """One pass of the oracle over the row slices [0:rows) of every workload (inputs made
    once, outside the timing); returns (flops, wall seconds)."""
    f, t, _, _ = _oracle_sample(0.0, rows, chunks=1)
    return f, t


def cpu_baseline(seconds):
    """The oracle as it stands on the host cores: the same sample (row slices [0:64) of every
    workload, same seeded inputs) timed with all cores and with one thread, wall clock,
    median of 3 runs each; plus a longer all-core sample of about `seconds`."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    rows = 64
    _oracle_pass(rows)  # inputs generated and caches warm before the timed runs
    runs_all = [_oracle_pass(rows) for _ in range(3)]
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            runs_one = [_oracle_pass(rows) for _ in range(3)]
        one_threads = 1
    except Exception:
        runs_one, one_threads = [], None
    flops = runs_all[0][0]
    t_all = statistics.median(t for _, t in runs_all)
    out = {"value": round(flops / t_all / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
           "sample": (f"oracle (numpy/scipy fp64) on row slices [0:{rows}) of every workload "
                      f"({flops / 1e9:.2f} GFLOP), wall clock, median of 3 runs; all {cores} host cores "
                      f"(nproc) for BLAS"),
           "all_cores_s": round(t_all, 3)}
    if runs_one:
        t_one = statistics.median(t for _, t in runs_one)
        out["single_thread"] = {"value": round(flops / t_one / 1e12, 6), "unit": "TFLOP/s", "threads": one_threads,
                                "s": round(t_one, 3)}
    f_long, t_long, _, desc = _oracle_sample(seconds)
    out["long_sample"] = {"value": round(f_long / t_long / 1e12, 6), "sample": desc}
    return out


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # steps x warmup of bounded oracle samples; the whole run stays within minutes
    per_step = max(0.05, min(6.0, 60.0 / max(1, args.steps + args.warmup)))
    rows = 64 if per_step >= 0.5 else 16  # short steps: one pass of 16-row slices (about 0.04 s)
    for _ in range(args.warmup):
        _oracle_sample(per_step / 4, rows)
    tot_f, tot_t, cores, desc = 0.0, 0.0, 1, ""
    for _ in range(args.steps):
        f, t, cores, desc = _oracle_sample(per_step, rows)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(SUITE), "parallelism": "host cores",
                       "sample": "row slices of every workload, about 0.05-6 s of oracle work per step"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc + f"; per step about {per_step:.1f} s"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """Launch one workload (or one HBM-bound kernel of hbm_runs) warm-up + steps times and
    exit: a small, fixed program for ncu."""
    import torch
    import gemm_bias_activation_tcgen05_b200 as fl
    torch.cuda.set_device(0)
    if args.profile in HBM_KERNELS:
        fn, _ = hbm_runs(fl, torch.cuda.current_stream().cuda_stream)[args.profile]
        for _ in range(args.warmup + args.steps):
            fn()
        torch.cuda.synchronize()
        return
    global SUITE
    SUITE = [args.profile]
    suite = Suite(fl, seed=0)
    sh = torch.cuda.current_stream().cuda_stream
    for _ in range(args.warmup + args.steps):
        for it in suite.items:
            suite.run_item(it, sh)
    torch.cuda.synchronize()
    suite.check()
    for it in suite.items:
        for p in it["plans"]:
            p.free()


def main():
    args = parse()
    if args.profile:
        run_profile(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
