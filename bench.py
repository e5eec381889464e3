#!/usr/bin/env python
"""Throughput of the NVFP4 + LoRA GEMM on B200, against its roofline, with the CPU oracle
timed beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cfg3] [--impl ours|reference]

One step = one pass of the workload's path over one batch: on the prepared path the in-place
refold of the adapter and the GEMM (two kernels), on the raw path one GEMM call.  The default
workload is cfg3, the large MLP-up shape M=8192, N=28672, K=8192, r=64 on the prepared path,
reported in TFLOPS against the dense FP4 peak; the same run then times the decode shape cfg1
(M=16, N=4096, K=4096, r=64, raw path + bias), reported in HBM GB/s, as a secondary block of the
same JSON line.  Inputs are rotated through enough copies (>= 3x the L2 size in total) that
every step reads them from HBM; steps are CUDA-graph replays timed with CUDA events on the
launching stream.  N > 1 (torchrun): every rank runs its own independent problem (weak scaling,
no collective on the data path); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "NVFP4+LoRA GEMM TFLOPS and % of FP4 tensor peak (HBM GB/s % at M<=16)"
PROFILES = os.path.join(ROOT, "profiles")

# workload name -> (config key or explicit dict, path, default steps)
WORKLOADS = {
    "cfg0": dict(src="cfg0", steps=2000),
    "cfg1": dict(src="cfg1", steps=20000),
    "cfg2": dict(src="cfg2", steps=2000),
    "cfg3": dict(src="cfg3", steps=100),
    "cfg4": dict(src=None, steps=None),   # adapter-switch sweep (its own runner)
    "quant": dict(src=None, steps=400),   # the NVFP4 quantizer on the cfg3 activations (its own runner)
    "moe": dict(src=None, steps=200),     # the grouped call on an 8-expert layer (its own runner)
    "bgmv": dict(src=None, steps=2000),   # the routed-MoE FC2 LoRA delta on a decode batch (its own runner)
}

QUANT_ROWS, QUANT_K = 8192, 8192         # cfg3's a: M x K

# the workload timed after the headline one in the same run (its own block in the line)
SECONDARY = {"cfg3": "cfg1"}


def describe(name):
    from workloads import CFG4, CONFIGS
    if name == "quant":
        return dict(rows=QUANT_ROWS, K=QUANT_K, seed=5)
    if name == "cfg4":
        # the sweep's headline point (the reference arm times the oracle on it)
        return dict(M=CFG4["Ms"][0], N=CFG4["N"], K=CFG4["K"], r=CFG4["rs"][0], path="raw",
                    alpha=CFG4["alpha"], lora_scale=1.0, bias=False, seed=CFG4["seed"])
    c = dict(CONFIGS[WORKLOADS[name]["src"]])
    return c


def upload_graph(g, stream) -> bool:
    """cudaGraphUpload of an instantiated graph on the launching stream, so that the first replay
    inside a timed region does not include uploading its nodes to the device (for a graph of 2000
    decode calls that first replay took about 3.5 ms longer).  No work of the graph runs.  Returns
    whether the upload succeeded."""
    import ctypes
    try:
        lib = ctypes.CDLL("libcudart.so.12")
        fn = lib.cudaGraphUpload
    except (OSError, AttributeError):
        return False
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    try:
        handle = int(g.raw_cuda_graph_exec())
    except (TypeError, ValueError, RuntimeError):
        return False
    return fn(ctypes.c_void_p(handle), ctypes.c_void_p(stream.cuda_stream)) == 0


def hold_device(stream, us=1000.0):
    """Enqueue a short spin on `stream` (PyTorch's own sleep kernel, outside any timed region) so
    that the start event recorded after it is timestamped only once the host has finished
    submitting the graph that follows: the timed region then holds the graph's kernels alone, not
    the host's launch latency (about 20 us for a 20-call graph, a quarter of a 20-call cfg1
    region).  Clock rate ~2 GHz; the spin length needs no precision."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2000))


def time_graph(step, n, stream, device, warm=3):
    """Capture n back-to-back calls of step(i) in one CUDA graph and time one replay with CUDA
    events on the launching stream (after an untimed warm-up replay).  Returns ms per call."""
    return time_graphs({"x": step}, n, stream, device, warm=warm, rounds=1)["x"]


def time_graphs(steps, n, stream, device, warm=3, rounds=3):
    """Like time_graph for several step functions at once: each is captured in its own graph of n
    calls, and the graphs are replayed in turn `rounds` times, so clock and temperature drift falls
    on all of them alike.  Returns the median ms per call of each."""
    graphs = {}
    with torch.cuda.stream(stream):
        for name, step in steps.items():
            for i in range(warm):
                step(i)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(i)
            graphs[name] = g
    for g in graphs.values():
        g.replay()
    torch.cuda.synchronize(device)
    times = {name: [] for name in steps}
    for _ in range(rounds):
        for name, g in graphs.items():
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            hold_device(stream)
            with torch.cuda.stream(stream):
                start.record(stream)
                g.replay()
                end.record(stream)
            torch.cuda.synchronize(device)
            times[name].append(start.elapsed_time(end) / n)
    del graphs
    return {name: sorted(v)[len(v) // 2] for name, v in times.items()}


def algorithmic(c):
    """Algorithmic bytes and flops of one call (padded scale rows and operand re-reads are
    implementation overhead and excluded)."""
    M, N, K, r = c["M"], c["N"], c["K"], c["r"]
    nbytes = (M * K // 2 + N * K // 2 + M * K // 16 + N * K // 16 + M * r * 2 + N * r * 2
              + (N * 2 if c["bias"] else 0) + M * N * 2 + 4 + 4)
    return nbytes, 2 * M * N * K, 2 * M * N * r


def max_over_ranks(value: float, device=None) -> float:
    """The slowest rank's time: every rank contributes its own, all receive the maximum."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job(per_rank_value: float, world: int) -> float:
    """Weak scaling: every rank processes the same amount of work in the (max-over-ranks) time,
    so the whole-job throughput is the per-rank throughput times the number of ranks."""
    return per_rank_value * world


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return j, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_hash(kernel="gemm"):
    """Hash of the kernel sources a recorded ncu figure depends on: the GEMM kernels (tiled, SM-pair,
    decode), the fold and the PTX wrappers for `gemm`, the quantizer and the wrappers for
    `quantize`, the LoRA-delta kernel and the headers it includes for `bgmv_delta`.  The host launcher is not hashed: a change of a launch configuration there is
    re-captured by hand."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "nvfp4_block_scaled_mm_b200", "csrc")
    if kernel == "quantize":
        files = ["ptx.cuh", "quantize.cuh"]
    elif kernel == "bgmv_delta":
        files = ["bgmv.cuh", "fold.cuh", "ptx.cuh"]
    else:
        files = ["fold.cuh", "gemm.cuh", "gemm_decode.cuh", "gemm_pair.cuh", "ptx.cuh"]
    for f in files:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel="gemm"):
    """DRAM bytes per launch of the workload's dominant kernel (`gemm` or `quantize`) from the
    committed ncu summary, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(PROFILES, f"{kernel}_{workload}_traffic.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha") != source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.01):
        self.ok = False
        self.samples = []
        self.reasons = 0
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def run_ours(args, workload, rank, world, device):
    """Time `workload` (cfg0..cfg3): K steps in one CUDA graph on the device, then (outside the
    timed region) the LoRA overhead against adapter-off and, on the prepared path, the raw path of
    the same inputs, then the end-to-end run through the public API with host buffers."""
    import nvfp4_block_scaled_mm_b200 as L
    from workloads import make_problem

    c = describe(workload)
    M, N, K, r = c["M"], c["N"], c["K"], c["r"]
    p = make_problem(M, N, K, r, c["seed"] + 1000 * rank, alpha=c["alpha"], lora_scale=c["lora_scale"],
                     bias=c["bias"])
    nbytes, flops, lora_flops = algorithmic(c)
    in_bytes = sum(t.numel() * t.element_size() for t in (p.a, p.b, p.a_sf, p.b_sf, p.d, p.lora_b)) + \
        (p.bias.numel() * 2 if p.bias is not None else 0)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(1, math.ceil(3 * l2 / in_bytes))

    def dev(t):
        return None if t is None else t.to(device)

    sets = []
    for _ in range(copies):
        sets.append(dict(a=dev(p.a), b=dev(p.b), a_sf=dev(p.a_sf), b_sf=dev(p.b_sf), d=dev(p.d),
                         lora_b=dev(p.lora_b), bias=dev(p.bias)))
    alpha = torch.tensor([c["alpha"]], dtype=torch.float32, device=device)
    s = torch.tensor([c["lora_scale"]], dtype=torch.float32, device=device)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    prepared = c["path"] == "prepared"
    adapters = []
    if prepared:
        for st in sets:
            adapters.append(L.prepare_nvfp4_lora_adapter(st["lora_b"], s, alpha))

    def step(i):
        st = sets[i % copies]
        if prepared:
            adp = adapters[i % copies]
            L.prepare_nvfp4_lora_adapter(st["lora_b"], s, alpha, out=adp)
            L.mm_nvfp4_lora(st["a"], st["b"], st["a_sf"], st["b_sf"], alpha, st["d"], lora_adapter=adp,
                            bias=st["bias"], out=out)
        else:
            L.mm_nvfp4_lora(st["a"], st["b"], st["a_sf"], st["b_sf"], alpha, st["d"], st["lora_b"], s,
                            bias=st["bias"], out=out)

    K_steps = args.steps if args.steps is not None else WORKLOADS[workload]["steps"]
    W = args.warmup
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(max(W, 3)):      # eager warm-up (also sets kernel attributes)
            step(i)
        L.nvfp4lora_device_status(stream)
        g_warm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_warm, stream=stream):
            for i in range(max(W, 3)):
                step(i)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(K_steps):
                step(i)
    launches_per_step = 2 if prepared else 1

    torch.cuda.synchronize(device)
    uploaded = upload_graph(g, stream)
    g_warm.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        hold_device(stream)
        with torch.cuda.stream(stream):
            start.record(stream)
            g.replay()
            end.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    L.nvfp4lora_device_status(stream)
    if world > 1:
        ms = max_over_ranks(ms, device)
    ms_step = ms / K_steps
    del g, g_warm

    # LoRA overhead (outside the timed region): the step, the same calls without an adapter, and
    # on the prepared path the GEMM alone with the adapter already folded and the raw path of the
    # same inputs, timed in turn so that clock drift falls on all of them alike.  At least ~20 ms
    # of work per graph, so that short steps are not dominated by the graph's edges.
    n_extra = max(K_steps, min(2000, int(math.ceil(0.02 / max(ms_step * 1e-3, 1e-7)))))

    def step_off(i):
        st = sets[i % copies]
        L.mm_nvfp4_lora(st["a"], st["b"], st["a_sf"], st["b_sf"], alpha, bias=st["bias"], out=out)

    kinds = {"path": step, "off": step_off}
    if prepared:
        def step_gemm(i):
            st = sets[i % copies]
            L.mm_nvfp4_lora(st["a"], st["b"], st["a_sf"], st["b_sf"], alpha, st["d"],
                            lora_adapter=adapters[i % copies], bias=st["bias"], out=out)

        def step_raw(i):
            st = sets[i % copies]
            L.mm_nvfp4_lora(st["a"], st["b"], st["a_sf"], st["b_sf"], alpha, st["d"], st["lora_b"], s,
                            bias=st["bias"], out=out)
        kinds["gemm"] = step_gemm
        kinds["raw"] = step_raw
    t = time_graphs(kinds, n_extra, stream, device)
    overhead = {"off_ms_per_call": t["off"], "path_ms_per_step": t["path"],
                "path_vs_off": t["path"] / t["off"] - 1.0, "calls": n_extra,
                "method": "median of 3 interleaved replays of one graph of %d calls each" % n_extra}
    if prepared:
        overhead["gemm_ms_per_call"] = t["gemm"]
        overhead["gemm_vs_off"] = t["gemm"] / t["off"] - 1.0
        overhead["raw_ms_per_call"] = t["raw"]
        overhead["raw_vs_off"] = t["raw"] / t["off"] - 1.0
    L.nvfp4lora_device_status(stream)

    # end to end through the public API with host buffers: per step, the activation-side
    # inputs (a, a_sf, d) go host -> device and the output comes back device -> host.
    e2e = run_e2e(L, p, sets, alpha, s, out, c, device, stream, min(K_steps, 2000), prepared,
                  adapters if prepared else None)
    if world > 1:
        e2e["ms_step"] = max_over_ranks(e2e["ms_step"], device)

    return dict(c=c, workload=workload, ms=ms, ms_step=ms_step, K=K_steps, W=max(W, 3), nbytes=nbytes,
                flops=flops, uploaded=uploaded, lora_flops=lora_flops, copies=copies, clocks=clk.summary(),
                e2e=e2e, launches=K_steps * launches_per_step, in_bytes=in_bytes, l2=l2, p=p,
                overhead=overhead)


def roofline_block(c, workload, value, unit, nbytes, ms_total):
    """The roofline of the workload's dominant kernel.  HBM-bound workloads: the measured copy
    bandwidth.  Tensor-bound ones: the dense FP4 peak derived from the measured cuBLAS bf16 GEMM
    (x 4, the nominal FP4 / bf16 ratio of 9 / 2.25 PFLOP/s), its burst figure for a timed region
    under two seconds and its sustained figure for a longer one."""
    peaks, peak_src = measured_peaks()
    if unit == "GB/s":
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": value, "peak": peak, "unit": "GB/s", "frac": value / peak,
                "peak_source": f"hbm_gbs of {peak_src}"}
    else:
        sustained = ms_total >= 2000.0 and "bf16_tflops_sustained" in peaks
        bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        peak = bf16 * 4.0
        which = "bf16_tflops_sustained" if sustained else "bf16_tflops (burst; timed region %.0f ms)" % ms_total
        roof = {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                "peak_source": f"{which} x 4 (nominal fp4/bf16) of {peak_src}"}
    roof["traffic"] = recorded_traffic(workload)
    roof["algorithmic_bytes_per_launch"] = nbytes
    return roof


def workload_line(args, res, world):
    """The JSON fields of one measured workload (the headline line, or a secondary block)."""
    c = res["c"]
    value, unit = metric_value(c, res["nbytes"], res["flops"], res["ms_step"])
    e2e = res["e2e"]
    e2e_val, e2e_unit = metric_value(c, res["nbytes"], res["flops"], e2e["ms_step"])
    line = {
        "value": whole_job(value, world), "unit": unit, "steps": res["K"], "warmup": res["W"],
        "ms_per_step": res["ms_step"],
        "config": config_block(args, c, res["workload"]),
        "roofline": roofline_block(c, res["workload"], value, unit, res["nbytes"], res["ms"]),
        "clocks": res["clocks"],
        "e2e": {"value": whole_job(e2e_val, world), "unit": e2e_unit, "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["ms_step"], "steps": e2e["steps"],
                "note": "per step: a, a_sf, d host->device (pinned, one staging buffer), call, out device->host; "
                        "step slots (4, or 2 for outputs over 64 MB) pipelined over three streams; the steps "
                        "captured in one CUDA graph; weights resident in HBM, rotating through the same copies "
                        "as the device-timed loop"},
        "gpu_launches": res["launches"],
        "lora_flops_per_step": res["lora_flops"], "tflops": res["flops"] / (res["ms_step"] * 1e-3) / 1e12,
        "gbs": res["nbytes"] / (res["ms_step"] * 1e-3) / 1e9, "weight_copies": res["copies"],
        "lora_overhead": res["overhead"],
    }
    ov = res["overhead"]
    if ov["calls"] >= 4 * res["K"]:
        # the same step in the longer graphs of the overhead replays, without the start-up share
        # that a short timed region carries (one rank's figure; the line's value stays the timed
        # region's)
        lv, lu = metric_value(c, res["nbytes"], res["flops"], ov["path_ms_per_step"])
        line["long_graph"] = {"calls": ov["calls"], "ms_per_step": ov["path_ms_per_step"], "value": lv, "unit": lu,
                              "frac": lv / line["roofline"]["peak"]}
    if "raw_ms_per_call" in ov:
        # the raw path of the same inputs (the workload names it for comparison)
        rv, ru = metric_value(c, res["nbytes"], res["flops"], ov["raw_ms_per_call"])
        line["raw_path"] = {"value": rv, "unit": ru, "ms_per_call": ov["raw_ms_per_call"],
                            "frac": rv / line["roofline"]["peak"], "vs_off": ov["raw_vs_off"]}
    return line


def cfg4_point(L, M, r, device, stream, l2, e2e=False):
    """One point of the adapter-switch sweep: N=14336, K=4096, 8 adapters switched every call.
    Times, each as a CUDA graph of back-to-back calls: the raw path with a different adapter's
    pointers per call; the prepared path refolding the next adapter inside the graph (fold +
    GEMM per call); and the prepared path with the next adapter's lora_b / lora_scale copied into
    fixed captured sources before the refold."""
    from workloads import CFG4, make_adapters, make_problem
    N, K = CFG4["N"], CFG4["K"]
    p = make_problem(M, N, K, r, CFG4["seed"] + 10 * M + r, alpha=CFG4["alpha"], lora_scale=1.0, bias=False)
    w_bytes = p.b.numel() + p.b_sf.numel()
    copies = max(1, math.ceil(3 * l2 / w_bytes))
    weights = [(p.b.to(device), p.b_sf.to(device)) for _ in range(copies)]
    a, a_sf, d = p.a.to(device), p.a_sf.to(device), p.d.to(device)
    adps = [(lb.to(device), torch.tensor([sv], dtype=torch.float32, device=device))
            for lb, sv in make_adapters(N, r, CFG4["adapters"], CFG4["seed"] + r)]
    alpha = torch.tensor([CFG4["alpha"]], dtype=torch.float32, device=device)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    c = dict(M=M, N=N, K=K, r=r, bias=False)
    nbytes, flops, _ = algorithmic(c)
    est = max(nbytes / 3e12, flops / 2e15)
    n = max(50, min(2000, int(0.03 / est)))
    na = len(adps)

    def step_raw(i):
        b, b_sf = weights[i % copies]
        lb, sv = adps[i % na]
        L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, d, lb, sv, out=out)

    adp = L.prepare_nvfp4_lora_adapter(adps[0][0], adps[0][1], alpha)

    def step_refold(i):
        b, b_sf = weights[i % copies]
        lb, sv = adps[i % na]
        L.prepare_nvfp4_lora_adapter(lb, sv, alpha, out=adp)
        L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, d, lora_adapter=adp, out=out)

    src_lb = adps[0][0].clone()
    src_s = adps[0][1].clone()
    adp2 = L.prepare_nvfp4_lora_adapter(src_lb, src_s, alpha)

    def step_copy(i):
        b, b_sf = weights[i % copies]
        lb, sv = adps[i % na]
        src_lb.copy_(lb)
        src_s.copy_(sv)
        L.prepare_nvfp4_lora_adapter(src_lb, src_s, alpha, out=adp2)
        L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, d, lora_adapter=adp2, out=out)

    res = dict(M=M, r=r, calls=n, weight_copies=copies, algorithmic_bytes=nbytes, flops=flops)
    for name, fn in (("raw_swap", step_raw), ("prepared_refold", step_refold), ("prepared_copy_refold", step_copy)):
        ms = time_graph(fn, n, stream, device)
        res[name] = {"us_per_call": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9, "tflops": flops / (ms * 1e-3) / 1e12}
    L.nvfp4lora_device_status(stream)
    if e2e:
        # the raw swap end to end: a, a_sf and d from pinned host memory, out back, weights and
        # adapters rotating as in the device-timed graph
        sets = [dict(b=weights[i % copies][0], b_sf=weights[i % copies][1], lora_b=adps[i % na][0],
                     s=adps[i % na][1], bias=None) for i in range(max(copies, na))]
        e = run_e2e(L, p, sets, alpha, None, out, c, device, stream, min(n, 2000), False, None)
        res["e2e"] = {"value": nbytes / (e["ms_step"] * 1e-3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                      "ms_per_step": e["ms_step"], "steps": e["steps"]}
    return res


def run_cfg4(args, rank, world, device):
    """The adapter-switch sweep (M x r grid).  The line's value is the raw path's HBM throughput
    at the decode point (M=1, r=8); every point is listed under "sweep"."""
    import nvfp4_block_scaled_mm_b200 as L
    from workloads import CFG4
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    stream = torch.cuda.Stream(device)
    sweep = []
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        for M in CFG4["Ms"]:
            for r in CFG4["rs"]:
                sweep.append(cfg4_point(L, M, r, device, stream, l2, e2e=not sweep))
                torch.cuda.empty_cache()
    head = sweep[0]
    ms = head["raw_swap"]["us_per_call"] * 1e-3
    if world > 1:
        ms = max_over_ranks(ms, device)
    value = head["algorithmic_bytes"] / (ms * 1e-3) / 1e9
    peaks, peak_src = measured_peaks()
    line = {
        "metric": METRIC, "value": whole_job(value, world), "unit": "GB/s", "n_gpus": world, "steps": head["calls"],
        "warmup": 3, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x ue4m3 -> fp32) + bf16 LoRA", "data": "synthetic",
        "config": {"workload": f"cfg4: adapter-switch sweep N={CFG4['N']} K={CFG4['K']} M in {list(CFG4['Ms'])} "
                               f"r in {list(CFG4['rs'])}, {CFG4['adapters']} adapters switched every call; "
                               f"value = raw path at M=1 r=8",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2_defeat": "weights rotate through copies totalling >= 3x L2",
                   "timing": "CUDA graph of back-to-back calls per point, CUDA events on the launching stream"},
        "roofline": {"bound": "hbm", "achieved": value, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": value / peaks["hbm_gbs"], "peak_source": f"hbm_gbs of {peak_src}", "traffic": None},
        "clocks": clk.summary(),
        "e2e": {"value": whole_job(head["e2e"]["value"], world), "unit": "GB/s",
                "h2d_bytes_per_step": head["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": head["e2e"]["d2h_bytes_per_step"],
                "ms_per_step": head["e2e"]["ms_per_step"], "steps": head["e2e"]["steps"],
                "method": "raw swap at M=1 r=8 through mm_nvfp4_lora: a, a_sf, d copied from pinned host memory "
                          "and out copied back every step; four step slots on three streams, one CUDA graph"},
        # this library's kernels per call: raw 1; refold + GEMM 2 (the copy_ kernels are PyTorch's)
        "gpu_launches": sum(pt["calls"] * k for pt in sweep for k in (1, 2, 2)),
        "sweep": sweep,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the headline point (M=1, r=8, raw path), as the reference arm times it
        from workloads import make_problem
        c = describe("cfg4")
        p = make_problem(c["M"], c["N"], c["K"], c["r"], c["seed"], alpha=c["alpha"],
                         lora_scale=c["lora_scale"], bias=c["bias"])
        nb, fl, _ = algorithmic(c)
        line["cpu_baseline"] = cpu_baseline(p, c, nb, fl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def moe_algorithmic(mp):
    """Algorithmic bytes and flops of one grouped call (rows past m_indptr[E] are not touched)."""
    E = mp.b.shape[0]
    used = int(mp.m_indptr[-1])
    N, K, r = mp.N, mp.K, mp.r
    nbytes = (used * K // 2 + E * N * K // 2 + used * K // 16 + E * N * K // 16 + used * r * 2 + E * N * r * 2
              + (E * N * 2 if mp.bias is not None else 0) + used * N * 2 + 4 * E + 4 * (E + 1) + 4)
    return nbytes, 2 * used * N * K


def moe_oracle_sample(mp, ncols):
    """The oracle's raw call form on expert 0's first 128 rows x the first `ncols` columns (the same
    definition the grouped form applies per segment); returns the fraction of the layer's outputs."""
    import oracle as O
    from workloads import MOE
    K, N, r = mp.K, mp.N, mp.r
    rows = 128
    sfb = O.sf_buffer_bytes(N, K)
    O.round_output(O.mm_raw(mp.a.numpy()[:rows], mp.b.numpy()[0], mp.a_sf.numpy()[:rows * K // 16],
                            mp.b_sf.numpy()[:sfb], float(mp.alpha[0]),
                            mp.d.view(torch.int16).numpy().view(np.uint16)[:rows],
                            mp.lora_b.view(torch.int16).numpy().view(np.uint16)[0], MOE["lora_scale"],
                            None if mp.bias is None else mp.bias.view(torch.int16).numpy().view(np.uint16)[0],
                            rows, N, K, r, cols=np.arange(ncols)))
    return rows * ncols / (int(mp.m_indptr[-1]) * N)


def moe_cpu_value(mp, budget_s):
    """Oracle throughput (TFLOPS) on bounded samples for about budget_s seconds, and the sample text."""
    _, flops = moe_algorithmic(mp)
    ncols = 64
    t0 = time.perf_counter()
    moe_oracle_sample(mp, ncols)
    dt = max(time.perf_counter() - t0, 1e-4)
    ncols = max(8, min(mp.N, int(ncols * budget_s / 3 / dt)))
    t0 = time.perf_counter()
    reps, frac = 0, 0.0
    while True:
        frac += moe_oracle_sample(mp, ncols)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 50:
            break
    dt = time.perf_counter() - t0
    value = flops * frac / dt / 1e12
    return value, (f"{reps} x oracle raw call form on expert 0's first 128 rows x the first {ncols} of {mp.N} "
                   f"columns ({frac / reps:.5f} of the layer each), {dt:.1f} s"), dt


def run_moe(args, rank, world, device):
    """The grouped call on an 8-expert layer (workloads.MOE): raw path with per-expert bias, inputs
    rotated through copies totalling >= 3x L2, K calls in one CUDA graph timed with CUDA events."""
    import nvfp4_block_scaled_mm_b200 as L
    from workloads import MOE, make_grouped_problem
    mp = make_grouped_problem(list(MOE["segments"]), MOE["N"], MOE["K"], MOE["r"], MOE["seed"] + 1000 * rank,
                              pad_rows=0)
    nbytes, flops = moe_algorithmic(mp)
    names = ("m_indptr", "a", "b", "a_sf", "b_sf", "alpha", "d", "lora_b", "bias")
    in_bytes = sum(getattr(mp, k).numel() * getattr(mp, k).element_size() for k in names)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(1, math.ceil(3 * l2 / in_bytes))
    sets = [{k: getattr(mp, k).to(device) for k in names} for _ in range(copies)]
    s = torch.tensor([MOE["lora_scale"]], dtype=torch.float32, device=device)
    out = torch.empty((mp.rows, mp.N), dtype=torch.bfloat16, device=device)

    def step(i):
        t = sets[i % copies]
        L.grouped_mm_nvfp4_lora(t["a"], t["b"], t["a_sf"], t["b_sf"], t["m_indptr"], t["alpha"], t["d"],
                                t["lora_b"], s, bias=t["bias"], out=out)

    steps = args.steps if args.steps is not None else WORKLOADS["moe"]["steps"]
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i)
        L.nvfp4lora_device_status(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                step(i)
    upload_graph(g, stream)
    g.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        hold_device(stream)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    L.nvfp4lora_device_status(stream)
    ms_total = e0.elapsed_time(e1)
    if world > 1:
        ms_total = max_over_ranks(ms_total, device)
    ms = ms_total / steps
    del g
    value = flops / (ms * 1e-3) / 1e12
    e2e = run_moe_e2e(L, mp, sets, s, device, min(steps, 200))
    if world > 1:
        e2e["ms_step"] = max_over_ranks(e2e["ms_step"], device)
    roof = roofline_block(None, "moe", value, "TFLOPS", nbytes, ms_total)
    line = {
        "metric": METRIC, "value": whole_job(value, world), "unit": "TFLOPS", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (e2m1 x ue4m3 -> fp32) + bf16 LoRA", "data": "synthetic",
        "config": {"workload": f"moe: grouped call, {len(MOE['segments'])} experts with rows {list(MOE['segments'])}, "
                               f"N={MOE['N']} K={MOE['K']} r={MOE['r']}, raw path + per-expert bias",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2_defeat": "inputs rotate through copies totalling >= 3x L2",
                   "timing": "CUDA graph of K back-to-back calls (uploaded to the device before the timed region), "
                             "CUDA events on the launching stream"},
        "roofline": roof, "clocks": clk.summary(),
        "e2e": {"value": whole_job(flops / (e2e["ms_step"] * 1e-3) / 1e12, world), "unit": "TFLOPS",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["ms_step"],
                "steps": e2e["steps"],
                "method": "grouped_mm_nvfp4_lora on device buffers filled from pinned host memory each step (a, a_sf, "
                          "d, m_indptr), out copied back; two step slots on three streams, one CUDA graph"},
        "gpu_launches": steps, "tflops": value, "gbs": nbytes / (ms * 1e-3) / 1e9, "weight_copies": copies,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, _ = moe_cpu_value(mp, 12.0)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOPS", "cores": oracle_threads(), "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_moe_e2e(L, mp, sets, s, device, steps):
    """The grouped call end to end: each step copies the activation side (a, a_sf, d, m_indptr) host
    -> device from pinned memory and out back; two step slots alternate over three streams."""
    slots = 2
    act = ("a", "a_sf", "d", "m_indptr")
    host = [{k: getattr(mp, k).pin_memory() for k in act} for _ in range(slots)]
    dev_in = [{k: torch.empty_like(getattr(mp, k), device=device) for k in act} for _ in range(slots)]
    outs = [torch.empty((mp.rows, mp.N), dtype=torch.bfloat16, device=device) for _ in range(slots)]
    outs_h = [torch.empty((mp.rows, mp.N), dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    stream = torch.cuda.current_stream(device)
    n_ev = steps + 8
    ev_in = [torch.cuda.Event() for _ in range(n_ev)]
    ev_call = [torch.cuda.Event() for _ in range(n_ev)]
    ev_out = [torch.cuda.Event() for _ in range(n_ev)]
    work = torch.cuda.Stream(device)

    def one(i, first):
        k = i % slots
        with torch.cuda.stream(s_in):
            if i - first >= slots:
                s_in.wait_event(ev_call[i - slots])
            for name in act:
                dev_in[k][name].copy_(host[k][name], non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(work):
            work.wait_event(ev_in[i])
            if i - first >= slots:
                work.wait_event(ev_out[i - slots])
            w = sets[i % len(sets)]
            x = dev_in[k]
            L.grouped_mm_nvfp4_lora(x["a"], w["b"], x["a_sf"], w["b_sf"], x["m_indptr"], w["alpha"], x["d"],
                                    w["lora_b"], s, bias=w["bias"], out=outs[k])
            ev_call[i].record(work)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_call[i])
            outs_h[k].copy_(outs[k], non_blocking=True)
            ev_out[i].record(s_out)

    for i in range(4):
        one(i, 0)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=work):
        fork = torch.cuda.Event()
        fork.record(work)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for i in range(steps):
            one(i + 4, 4)
        for st_ in (s_in, s_out):
            join = torch.cuda.Event()
            join.record(st_)
            work.wait_event(join)
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(work):
        e0.record(work)
        g.replay()
        e1.record(work)
    torch.cuda.synchronize(device)
    L.nvfp4lora_device_status(work)
    ms = e0.elapsed_time(e1) / steps
    del g
    h2d = sum(getattr(mp, k).numel() * getattr(mp, k).element_size() for k in act)
    return dict(ms_step=ms, steps=steps, h2d=h2d, d2h=mp.rows * mp.N * 2)


def bgmv_workload_text():
    from workloads import BGMV
    return (f"bgmv: routed-MoE FC2 LoRA delta, T={BGMV['T']} tokens top-{BGMV['top_k']} of {BGMV['num_experts']} "
            f"experts, {BGMV['num_adapters']} adapters, I={BGMV['I']} H={BGMV['H']} rank={BGMV['rank']}, bf16")


def bgmv_algorithmic(bp):
    """Algorithmic bytes and flops of one delta call: the active slots' activation rows, every
    (adapter, expert) block pair that an active slot uses (A and B once each), the routing and
    pointer tables, and the output."""
    ids = bp.topk_ids.numpy()
    perm = bp.perm.numpy().reshape(bp.T, bp.top_k)
    lids = bp.lora_ids.numpy()
    pairs, rows = set(), 0
    for t in range(bp.T):
        if lids[t] < 0:
            continue
        for j in range(bp.top_k):
            if perm[t, j] >= 0:
                rows += 1
                pairs.add((int(lids[t]), int(ids[t, j])))
    el = 2
    nbytes = (rows * bp.I * el + len(pairs) * (bp.rank * bp.I + bp.H * bp.rank) * el + bp.T * bp.top_k * 12
              + bp.T * 4 + 2 * bp.num_experts * 8 + bp.T * bp.H * el)
    return nbytes, 2 * rows * (bp.rank * bp.I + bp.H * bp.rank)


def bgmv_cpu_value(bp, budget_s):
    """Oracle throughput (GB/s of the call's algorithmic bytes) on bounded token samples."""
    import oracle as O
    nbytes, _ = bgmv_algorithmic(bp)
    b16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    act, ab, bb = b16(bp.act), [b16(x) for x in bp.a_banks], [b16(x) for x in bp.b_banks]
    ntok = 8
    t0 = time.perf_counter()
    reps = 0
    while True:
        toks = np.arange(reps * ntok, (reps + 1) * ntok) % bp.T
        O.round_to(O.bgmv_moe_lora_delta(act, bp.perm.numpy(), ab, bp.stride_a, bb, bp.stride_b,
                                         bp.topk_ids.numpy(), bp.topk_weights.numpy(), bp.lora_ids.numpy(),
                                         bp.rank, bp.H, bp.scale, "bf16", tokens=toks), "bf16")
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 400:
            break
    dt = time.perf_counter() - t0
    frac = reps * ntok / bp.T
    return nbytes * frac / dt / 1e9, f"{reps} x oracle delta on {ntok} of {bp.T} tokens, {dt:.1f} s", dt


def run_bgmv(args, rank, world, device):
    """The routed-MoE FC2 LoRA delta on a decode batch (workloads.BGMV): memory-bound, reported in
    GB/s of algorithmic bytes against the measured HBM copy bandwidth.  Activations, banks and
    routing rotate through copies totalling >= 3x L2; K calls in one CUDA graph."""
    import nvfp4_block_scaled_mm_b200 as L
    from workloads import BGMV, make_bgmv_problem
    cfg = dict(BGMV)
    cfg["seed"] = BGMV["seed"] + 1000 * rank
    bp = make_bgmv_problem(**cfg)
    nbytes, flops = bgmv_algorithmic(bp)
    route = ("perm", "topk_ids", "topk_weights", "lora_ids")
    in_bytes = (bp.act.numel() * 2 + sum(x.numel() * 2 for x in bp.a_banks + bp.b_banks)
                + sum(getattr(bp, k).numel() * 4 for k in route))
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(1, math.ceil(3 * l2 / in_bytes))
    sets = []
    for _ in range(copies):
        a = [x.to(device) for x in bp.a_banks]
        b = [x.to(device) for x in bp.b_banks]
        sets.append(dict(act=bp.act.to(device), a=a, b=b, wa=L.fill_w_ptr(a), wb=L.fill_w_ptr(b),
                         **{k: getattr(bp, k).to(device) for k in route}))
    out = torch.empty((bp.T, bp.H), dtype=torch.bfloat16, device=device)

    def call(t, act, o):
        L.bgmv_moe_gemm2_lora_delta(act, t["perm"], t["wa"], bp.stride_a, t["wb"], bp.stride_b, t["topk_ids"],
                                    t["topk_weights"], t["lora_ids"], bp.rank, bp.H, scale=bp.scale, out=o)

    steps = args.steps if args.steps is not None else WORKLOADS["bgmv"]["steps"]
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            call(sets[i % copies], sets[i % copies]["act"], out)
        L.nvfp4lora_device_status(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                call(sets[i % copies], sets[i % copies]["act"], out)
    upload_graph(g, stream)
    g.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        hold_device(stream)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    L.nvfp4lora_device_status(stream)
    ms_total = e0.elapsed_time(e1)
    if world > 1:
        ms_total = max_over_ranks(ms_total, device)
    ms = ms_total / steps
    del g
    value = nbytes / (ms * 1e-3) / 1e9

    # end to end: the activation rows and the routing tables come from pinned host memory every step,
    # the delta goes back; the adapter banks stay resident (model state)
    slots = 4
    host = [dict(act=bp.act.pin_memory(), **{k: getattr(bp, k).pin_memory() for k in route}) for _ in range(slots)]
    dev_in = [{k: torch.empty_like(v, device=device) for k, v in h.items()} for h in host]
    outs = [torch.empty((bp.T, bp.H), dtype=torch.bfloat16, device=device) for _ in range(slots)]
    outs_h = [torch.empty((bp.T, bp.H), dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    s_in, s_out, work = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    e2e_steps = min(steps, 2000)
    n_ev = e2e_steps + 8
    ev_in = [torch.cuda.Event() for _ in range(n_ev)]
    ev_call = [torch.cuda.Event() for _ in range(n_ev)]
    ev_out = [torch.cuda.Event() for _ in range(n_ev)]

    def one(i, first):
        k = i % slots
        with torch.cuda.stream(s_in):
            if i - first >= slots:
                s_in.wait_event(ev_call[i - slots])
            for name, h in host[k].items():
                dev_in[k][name].copy_(h, non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(work):
            work.wait_event(ev_in[i])
            if i - first >= slots:
                work.wait_event(ev_out[i - slots])
            w = dict(sets[i % copies])
            w.update({name: dev_in[k][name] for name in route})
            call(w, dev_in[k]["act"], outs[k])
            ev_call[i].record(work)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_call[i])
            outs_h[k].copy_(outs[k], non_blocking=True)
            ev_out[i].record(s_out)

    for i in range(4):
        one(i, 0)
    torch.cuda.synchronize(device)
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=work):
        fork = torch.cuda.Event()
        fork.record(work)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for i in range(e2e_steps):
            one(i + 4, 4)
        for st_ in (s_in, s_out):
            join = torch.cuda.Event()
            join.record(st_)
            work.wait_event(join)
    ge.replay()
    torch.cuda.synchronize(device)
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(work):
        e2.record(work)
        ge.replay()
        e3.record(work)
    torch.cuda.synchronize(device)
    L.nvfp4lora_device_status(work)
    ms_e2e = e2.elapsed_time(e3) / e2e_steps
    del ge
    if world > 1:
        ms_e2e = max_over_ranks(ms_e2e, device)
    h2d = sum(v.numel() * v.element_size() for v in host[0].values())

    roof = roofline_block(None, "bgmv", value, "GB/s", nbytes, ms_total)
    roof["traffic"] = recorded_traffic("bgmv", "bgmv_delta")
    line = {
        "metric": METRIC, "value": whole_job(value, world), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 x bf16 -> fp32", "data": "synthetic",
        "config": {"workload": bgmv_workload_text(),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2_defeat": "activations, banks and routing rotate through copies totalling >= 3x L2",
                   "timing": "CUDA graph of K back-to-back calls (uploaded to the device before the timed region), "
                             "CUDA events on the launching stream"},
        "roofline": roof, "clocks": clk.summary(),
        "e2e": {"value": whole_job(nbytes / (ms_e2e * 1e-3) / 1e9, world), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": bp.T * bp.H * 2, "ms_per_step": ms_e2e,
                "steps": e2e_steps,
                "method": "bgmv_moe_gemm2_lora_delta with the activation rows and routing tables copied from pinned "
                          "host memory each step and the delta copied back; banks resident; four step slots on "
                          "three streams, one CUDA graph"},
        "gpu_launches": steps, "gflops": flops / (ms * 1e-3) / 1e9, "copies": copies,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, _ = bgmv_cpu_value(bp, 10.0)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_reference_bgmv(args):
    """Reference arm of the LoRA-delta workload: the oracle on a bounded token sample per step."""
    from workloads import BGMV, make_bgmv_problem
    bp = make_bgmv_problem(**BGMV)
    K_steps = args.steps if args.steps is not None else 20
    per_step = max(0.05, 120.0 / (K_steps + args.warmup))
    value, sample, dt = bgmv_cpu_value(bp, per_step * K_steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": K_steps, "warmup": args.warmup, "ms_per_step": dt / K_steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": bgmv_workload_text()},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_quant(args, rank, world, device):
    """The NVFP4 quantizer (fp4_quantize reading) on bf16 activations of cfg3's shape: HBM-bound,
    2 bytes read and 0.5 + 1/16 written per element.  Inputs rotate through copies totalling
    >= 3x L2; K calls in one CUDA graph, timed with CUDA events."""
    import nvfp4_block_scaled_mm_b200 as L
    rows, K = QUANT_ROWS, QUANT_K
    g = torch.Generator().manual_seed(5 + 1000 * rank)
    x = (torch.randn(rows, K, generator=g) * 2.0).to(torch.bfloat16)
    gs_v = 448.0 * 6.0 / x.float().abs().max().item()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(1, math.ceil(3 * l2 / (x.numel() * 2)))
    xs = [x.to(device) for _ in range(copies)]
    gs = torch.tensor([gs_v], dtype=torch.float32, device=device)
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((rows + 127) // 128 * 128 * (K // 16), dtype=torch.uint8, device=device)
    nbytes = rows * K * 2 + rows * K // 2 + scales.numel() + 4
    steps = args.steps if args.steps is not None else WORKLOADS["quant"]["steps"]
    stream = torch.cuda.Stream(device)

    def step(i):
        L.fp4_quantize(xs[i % copies], gs, codes=codes, scales=scales)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i)
        g_run = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_run, stream=stream):
            for i in range(steps):
                step(i)
    upload_graph(g_run, stream)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            g_run.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
    L.nvfp4lora_device_status(stream)
    ms = e0.elapsed_time(e1) / steps
    if world > 1:
        ms = max_over_ranks(ms, device)
    value = nbytes / (ms * 1e-3) / 1e9
    e2e = run_quant_e2e(L, x, gs, device, stream, min(steps, 50))
    if world > 1:
        e2e["ms_step"] = max_over_ranks(e2e["ms_step"], device)
    peaks, peak_src = measured_peaks()
    line = {
        "metric": METRIC, "value": whole_job(value, world), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 -> nvfp4 (e2m1 codes + ue4m3 scales)", "data": "synthetic",
        "config": {"workload": f"quant: NVFP4 quantizer, bf16 [{rows}, {K}] (cfg3's activations) -> codes + scales",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2_defeat": "inputs rotate through copies totalling >= 3x L2",
                   "timing": "CUDA graph of K back-to-back calls (uploaded to the device before the timed region), "
                      "CUDA events on the launching stream"},
        "roofline": {"bound": "hbm", "achieved": value, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": value / peaks["hbm_gbs"], "peak_source": f"hbm_gbs of {peak_src}",
                     "traffic": recorded_traffic("quant", kernel="quantize"), "algorithmic_bytes_per_launch": nbytes},
        "clocks": clk.summary(),
        "e2e": {"value": whole_job(nbytes / (e2e["ms_step"] * 1e-3) / 1e9, world), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": e2e["ms_step"], "steps": e2e["steps"],
                "method": "fp4_quantize on device buffers filled from pinned host memory each step, codes and "
                          "scales copied back; two step slots, copies and calls on three streams, one CUDA graph"},
        "gpu_launches": steps,
    }
    if rank == 0 and not args.no_cpu_baseline:
        import time
        import oracle as O
        xb = x[:64].view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < 10.0:
            O.quantize_nvfp4(xb, gs_v)
            n += 1
        dt = (time.perf_counter() - t0) / n
        frac = 64 / rows
        line["cpu_baseline"] = {"value": nbytes * frac / dt / 1e9, "unit": "GB/s", "cores": torch.get_num_threads(),
                                "kind": "oracle",
                                "sample": f"{n} x oracle quantizer on the first 64 of {rows} rows "
                                          f"({frac:.4f} of the workload each), {n * dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_quant_e2e(L, x, gs, device, stream, steps):
    """The quantizer end to end through fp4_quantize with host buffers: each step copies the bf16
    activations host -> device from pinned memory, quantizes, and copies the codes and scales back
    to pinned memory.  Two step slots alternate over three streams ordered by events (as in the
    GEMM's end-to-end run), replayed from one CUDA graph."""
    slots = 2
    rows, K = x.shape
    n_sf = (rows + 127) // 128 * 128 * (K // 16)
    host_x = [x.pin_memory() for _ in range(slots)]
    dev_x = [torch.empty_like(x, device=device) for _ in range(slots)]
    dev_c = [torch.empty((rows, K // 2), dtype=torch.uint8, device=device) for _ in range(slots)]
    dev_s = [torch.empty(n_sf, dtype=torch.uint8, device=device) for _ in range(slots)]
    host_c = [torch.empty((rows, K // 2), dtype=torch.uint8).pin_memory() for _ in range(slots)]
    host_s = [torch.empty(n_sf, dtype=torch.uint8).pin_memory() for _ in range(slots)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    n_ev = steps + 8
    ev_in = [torch.cuda.Event() for _ in range(n_ev)]
    ev_call = [torch.cuda.Event() for _ in range(n_ev)]
    ev_out = [torch.cuda.Event() for _ in range(n_ev)]

    def one(i, first):
        k = i % slots
        with torch.cuda.stream(s_in):
            if i - first >= slots:
                s_in.wait_event(ev_call[i - slots])
            dev_x[k].copy_(host_x[k], non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[i])
            if i - first >= slots:
                stream.wait_event(ev_out[i - slots])
            L.fp4_quantize(dev_x[k], gs, codes=dev_c[k], scales=dev_s[k])
            ev_call[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_call[i])
            host_c[k].copy_(dev_c[k], non_blocking=True)
            host_s[k].copy_(dev_s[k], non_blocking=True)
            ev_out[i].record(s_out)

    for i in range(4):
        one(i, 0)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fork = torch.cuda.Event()
        fork.record(stream)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for i in range(steps):
            one(i + 4, 4)
        for st_ in (s_in, s_out):
            join = torch.cuda.Event()
            join.record(st_)
            stream.wait_event(join)
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    L.nvfp4lora_device_status(stream)
    ms = e0.elapsed_time(e1) / steps
    del g
    return dict(ms_step=ms, steps=steps, h2d=x.numel() * 2, d2h=rows * K // 2 + n_sf)


def run_e2e(L, p, sets, alpha, s, out, c, device, stream, steps, prepared, adps, slots=None):
    """End to end through the public API with host buffers.  Every step copies its activation-side
    inputs (a, a_sf, d) host -> device from pinned memory, makes the call, and copies out back to
    pinned host memory.  a's, a_sf's and d's bytes sit in one pinned staging buffer (one copy per
    step).  The resident weights (b, b_sf, lora_b or the prepared adapter, bias) rotate through
    the same device copies as the device-timed loop, so they are read from HBM, not L2.  Steps are
    pipelined the way a serving loop would run them: step slots (four, or two for a
    large output) rotate, and the host -> device copies, the calls and the device -> host copies
    run on three streams ordered by events, so one step's copies overlap its neighbours' calls.  The timed steps are replayed
    from one CUDA graph."""
    def region(nbytes):
        return (nbytes + 255) // 256 * 256
    na, nsf, nd = p.a.numel(), p.a_sf.numel(), p.d.numel() * 2
    oa, osf, od = 0, region(na), region(na) + region(nsf)
    total = od + region(nd)
    # four steps in flight where a step's output is small (the copies are latency-bound: cfg1
    # runs 1231 GB/s with four slots against 1013 with two, and eight add nothing); two where
    # it is large, to bound the pinned host memory (cfg3: 470 MB per slot)
    slots = slots or (4 if out.numel() * 2 <= (64 << 20) else 2)
    host_in, dev_in, views = [], [], []
    for _ in range(slots):
        h = torch.empty(total, dtype=torch.uint8).pin_memory()
        h[oa:oa + na].copy_(p.a.reshape(-1))
        h[osf:osf + nsf].copy_(p.a_sf.reshape(-1))
        h[od:od + nd].copy_(p.d.reshape(-1).view(torch.uint8))
        dbuf = torch.empty(total, dtype=torch.uint8, device=device)
        host_in.append(h)
        dev_in.append(dbuf)
        views.append((dbuf[oa:oa + na].view(p.a.shape), dbuf[osf:osf + nsf].view(p.a_sf.shape),
                      dbuf[od:od + nd].view(torch.bfloat16).view(p.d.shape)))
    outs = [torch.empty_like(out) for _ in range(slots)]
    outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(slots)]
    h2d = na + nsf + nd
    d2h = out.numel() * 2
    pipelined = True
    if pipelined:
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    else:
        s_in = s_out = stream
    n_ev = steps + 8
    ev_in = [torch.cuda.Event() for _ in range(n_ev)]
    ev_call = [torch.cuda.Event() for _ in range(n_ev)]
    ev_out = [torch.cuda.Event() for _ in range(n_ev)]

    def one(i, first):
        # waits only on events of this batch of steps (a captured batch cannot wait on the others)
        k = i % slots if pipelined else 0
        with torch.cuda.stream(s_in):
            if pipelined and i - first >= slots:
                s_in.wait_event(ev_call[i - slots])     # the slot's previous call has read its inputs
            dev_in[k].copy_(host_in[k], non_blocking=True)
            if pipelined:
                ev_in[i].record(s_in)
        with torch.cuda.stream(stream):
            if pipelined:
                stream.wait_event(ev_in[i])
                if i - first >= slots:
                    stream.wait_event(ev_out[i - slots])    # the slot's previous output has been copied out
            a_d, a_sf_d, d_d = views[k]
            st = sets[i % len(sets)]
            if prepared:
                L.mm_nvfp4_lora(a_d, st["b"], a_sf_d, st["b_sf"], alpha, d_d, lora_adapter=adps[i % len(adps)],
                                bias=st["bias"], out=outs[k])
            else:
                L.mm_nvfp4_lora(a_d, st["b"], a_sf_d, st["b_sf"], alpha, d_d, st["lora_b"], st.get("s", s),
                                bias=st["bias"], out=outs[k])
            if pipelined:
                ev_call[i].record(stream)
        with torch.cuda.stream(s_out):
            if pipelined:
                s_out.wait_event(ev_call[i])
            outs_h[k].copy_(outs[k], non_blocking=True)
            if pipelined:
                ev_out[i].record(s_out)

    for i in range(4):
        one(i, 0)
    torch.cuda.synchronize(device)
    # the steps are captured in one CUDA graph (copies, calls, and on the pipelined path the
    # cross-stream orderings), so the host issues one launch instead of a Python loop per step
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        if pipelined:
            fork = torch.cuda.Event()
            fork.record(stream)
            s_in.wait_event(fork)
            s_out.wait_event(fork)
        for i in range(steps):
            one(i + 4, 4)
        if pipelined:
            for st_ in (s_in, s_out):
                join = torch.cuda.Event()
                join.record(st_)
                stream.wait_event(join)
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    del g
    return dict(ms_step=ms, steps=steps, h2d=h2d, d2h=d2h, pipelined=pipelined)


# ---------------------------------------------------------------------------------------
# the oracle as the CPU baseline / reference arm
# ---------------------------------------------------------------------------------------

def sample_rows(c):
    """Output rows of the oracle's bounded sample: all of them up to 256, else the first 256 (the
    oracle dequantises every sampled row of a on each call, so rows bound its fixed cost)."""
    return min(c["M"], 256)


def oracle_sample(p, c, ncols):
    """Oracle on the first `sample_rows(c)` rows x the first `ncols` output columns of the workload
    (the oracle's own call forms, restricted to those outputs); returns the fraction of the
    workload's outputs this covers."""
    import oracle as O
    a = p.a.numpy(); b = p.b.numpy(); a_sf = p.a_sf.numpy(); b_sf = p.b_sf.numpy()
    dbits = p.d.view(torch.int16).numpy().view(np.uint16)
    lbits = p.lora_b.view(torch.int16).numpy().view(np.uint16)
    bias = None if p.bias is None else p.bias.view(torch.int16).numpy().view(np.uint16)
    M, N, K, r = c["M"], c["N"], c["K"], c["r"]
    nrows = sample_rows(c)
    rows = np.arange(nrows)
    cols = np.arange(ncols)
    if c["path"] == "prepared":
        ratio, bf = O.fold(lbits, c["lora_scale"], c["alpha"])
        y = O.mm_prepared(a, b, a_sf, b_sf, c["alpha"], dbits, bf, ratio, bias, M, N, K, r, rows=rows, cols=cols)
    else:
        y = O.mm_raw(a, b, a_sf, b_sf, c["alpha"], dbits, lbits, c["lora_scale"], bias, M, N, K, r,
                     rows=rows, cols=cols)
    O.round_output(y)
    return nrows * ncols / (M * N)


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    return os.cpu_count()


def calibrate_cols(p, c, budget_s):
    ncols = min(c["N"], 64)
    t0 = time.perf_counter()
    oracle_sample(p, c, ncols)
    dt = max(time.perf_counter() - t0, 1e-4)
    want = int(ncols * budget_s / dt)
    return max(8, min(c["N"], want))


def cpu_baseline(p, c, nbytes, flops, budget_s=12.0):
    """Time the oracle on a bounded sample of the workload for about `budget_s` seconds."""
    ncols = calibrate_cols(p, c, budget_s / 3)
    t0 = time.perf_counter()
    reps = 0
    frac = 0.0
    while True:
        frac += oracle_sample(p, c, ncols)
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= 50:
            break
    dt = time.perf_counter() - t0
    value, unit = metric_value(c, nbytes * frac / reps, flops * frac / reps, dt / reps * 1e3)
    return dict(value=value, unit=unit, cores=oracle_threads(), kind="oracle",
                sample=f"{reps} x oracle on the first {sample_rows(c)} of {c['M']} rows x the first {ncols} of "
                       f"{c['N']} output columns ({frac / reps:.5f} of the workload each), {dt:.1f} s")


def metric_value(c, nbytes, flops, ms):
    if c["M"] <= 16:
        return nbytes / (ms * 1e-3) / 1e9, "GB/s"
    return flops / (ms * 1e-3) / 1e12, "TFLOPS"


def run_reference(args, rank, world):
    """The reference arm: the oracle, as it stands, timed on the host cores on the same
    workload, one bounded sample per step."""
    from workloads import make_problem
    if rank != 0:
        return 0
    if args.workload == "quant":
        return run_reference_quant(args)
    if args.workload == "moe":
        return run_reference_moe(args)
    if args.workload == "bgmv":
        return run_reference_bgmv(args)
    c = describe(args.workload)
    p = make_problem(c["M"], c["N"], c["K"], c["r"], c["seed"], alpha=c["alpha"],
                     lora_scale=c["lora_scale"], bias=c["bias"])
    nbytes, flops, _ = algorithmic(c)
    K_steps = args.steps if args.steps is not None else 20
    W = args.warmup
    per_step_budget = max(0.01, 120.0 / (K_steps + W))
    ncols = calibrate_cols(p, c, per_step_budget)
    for _ in range(W):
        oracle_sample(p, c, ncols)
    t0 = time.perf_counter()
    frac = 0.0
    for _ in range(K_steps):
        frac += oracle_sample(p, c, ncols)
    dt = time.perf_counter() - t0
    ms_step = dt / K_steps * 1e3
    value, unit = metric_value(c, nbytes * frac / K_steps, flops * frac / K_steps, ms_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": K_steps, "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(args, c),
        "cpu_baseline": {"value": value, "unit": unit, "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"each step: oracle on the first {sample_rows(c)} of {c['M']} rows x the first "
                                   f"{ncols} of {c['N']} output columns "
                                   f"({sample_rows(c) * ncols / (c['M'] * c['N']):.5f} of the workload)"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_moe(args):
    """Reference arm of the grouped workload: the oracle on a bounded sample per step."""
    from workloads import MOE, make_grouped_problem
    mp = make_grouped_problem(list(MOE["segments"]), MOE["N"], MOE["K"], MOE["r"], MOE["seed"], pad_rows=0)
    K_steps = args.steps if args.steps is not None else 20
    per_step = max(0.05, 120.0 / (K_steps + args.warmup))
    value, sample, dt = moe_cpu_value(mp, per_step * K_steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": K_steps, "warmup": args.warmup, "ms_per_step": dt / K_steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"moe: grouped call, {len(MOE['segments'])} experts with rows {list(MOE['segments'])}, "
                               f"N={MOE['N']} K={MOE['K']} r={MOE['r']}, raw path + per-expert bias"},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_quant(args):
    """Reference arm of the quantizer workload: the oracle quantizer on a bounded row sample."""
    import oracle as O
    c = describe("quant")
    rows, K = c["rows"], c["K"]
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(rows, K, generator=g) * 2.0).to(torch.bfloat16)
    gs_v = 448.0 * 6.0 / x.float().abs().max().item()
    nrows = 64
    xb = x[:nrows].view(torch.int16).numpy().view(np.uint16)
    nbytes = rows * K * 2 + rows * K // 2 + (rows + 127) // 128 * 128 * (K // 16) + 4
    K_steps = args.steps if args.steps is not None else 20
    for _ in range(args.warmup):
        O.quantize_nvfp4(xb, gs_v)
    t0 = time.perf_counter()
    for _ in range(K_steps):
        O.quantize_nvfp4(xb, gs_v)
    ms_step = (time.perf_counter() - t0) / K_steps * 1e3
    value = nbytes * nrows / rows / (ms_step * 1e-3) / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": K_steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"quant: NVFP4 quantizer, bf16 [{rows}, {K}] (cfg3's activations) -> codes + scales"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"each step: oracle quantizer on the first {nrows} of {rows} rows"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(args, c, workload=None):
    workload = workload or args.workload
    what = "fold + GEMM per step" if c["path"] == "prepared" else "one call per step"
    return {"workload": f"{workload}: M={c['M']} N={c['N']} K={c['K']} r={c['r']} {c['path']} path"
                        f"{' + bias' if c['bias'] else ''} ({what})",
            "M": c["M"], "N": c["N"], "K": c["K"], "r": c["r"], "path": c["path"],
            "alpha": c["alpha"], "lora_scale": c["lora_scale"], "bias": c["bias"],
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU",
            "l2_defeat": "weights and activations rotate through copies totalling >= 3x L2",
            "timing": "CUDA graph of K back-to-back calls (uploaded to the device before the timed region), "
                      "CUDA events on the launching stream"}


# ---------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="cfg3")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the secondary workload's block")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device,
                                             timeout=datetime.timedelta(seconds=120))
    if args.workload in ("cfg4", "quant", "moe", "bgmv"):
        rc = {"cfg4": run_cfg4, "quant": run_quant, "moe": run_moe, "bgmv": run_bgmv}[args.workload](
            args, rank, world, device)
        if world > 1:
            torch.distributed.destroy_process_group()
        return rc
    # the headline workload, then (default run only) the decode workload in the same process, so
    # that one driver run measures both regimes of the metric: TFLOPS / % of FP4 peak at large M
    # and HBM GB/s at M <= 16
    res = run_ours(args, args.workload, rank, world, device)
    head = workload_line(args, res, world)
    line = {"metric": METRIC, "value": head.pop("value"), "unit": head.pop("unit"), "n_gpus": world,
            "steps": head.pop("steps"), "warmup": head.pop("warmup"), "ms_per_step": head.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x ue4m3 -> fp32) + bf16 LoRA", "data": "synthetic"}
    line.update(head)
    secondary = SECONDARY.get(args.workload) if not args.no_secondary else None
    if secondary:
        torch.cuda.empty_cache()
        sec = run_ours(args, secondary, rank, world, device)
        line["secondary"] = {secondary: workload_line(args, sec, world)}
        line["gpu_launches"] += sec["launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(res["p"], res["c"], res["nbytes"], res["flops"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
