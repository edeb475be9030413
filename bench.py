#!/usr/bin/env python
"""Benchmark of libmlstm on B200: one JSON line on rank 0.

A step is one pass of the hot path over one batch of synthetic input: one
``mlstm_fwd`` (gate preprocessing, chunk-state carry, chunk outputs) over the
workload's B x S tokens.  The default workload is the long-context prefill,
B1 NH8 S131072 d256/512 chunk 128, the largest forward configuration that fits
one GPU.  ``value`` is tokens per second over the whole job (B x S tokens per
step per GPU), timed with CUDA events around exactly ``--steps`` graph replays,
the max over ranks.  Inputs live in HBM before the timed region; the input sets
used in rotation are each larger than the 126 MB L2.

The other workloads are timed beside it under ``workloads`` (the 2048- and
8192-token prefills, the decode step on a 1 GiB state, the sLSTM recurrence).

Heads and batches are independent, so N GPUs run N independent replicas of the
workload with no collective ("weak" scaling); the only collectives are the
barrier and the max of the timings.

``--impl reference`` times the fp64 CPU oracle (the plain recurrence) on a
bounded sample of the same workload instead, on rank 0 only.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from xlstm_mlstm_cell_b200 import binding  # noqa: E402
from xlstm_mlstm_cell_b200.workloads import WORKLOADS, Workload  # noqa: E402

METRIC = "mLSTM chunkwise fwd tokens/s + % TC peak; decode-step HBM GB/s"
DEFAULT_WORKLOAD = "fwd_bf16_long"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
FP32_LANES_PER_SM, N_SM = 128, 148
E2E_MAX_STEPS = 20          # steps of the end-to-end run (each moves GBs over PCIe)
REF_SAMPLE_TOKENS = 8192    # tokens per head of one reference-arm step (the oracle on the host cores)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------- algorithmic work

def segments(w: Workload) -> int:
    """Segments per head of the library's tensor-core path for the workload (its own planner)."""
    return binding.fwd_segments(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype)


def bytes_per_token_head(w: Workload) -> int:
    """Algorithmic HBM bytes per token and head: q, k, v (and o) read once, h written once and the
    two gate pre-activations read once, e (2 dk + dv) + e dv [o] + e dv + 8."""
    e = 4 if w.dtype == "f32" else 2
    return e * (2 * w.DHQK + w.DHV) + (e * w.DHV if w.ogate else 0) + e * w.DHV + 8


def flops_per_token_head(w: Workload) -> int:
    """Algorithmic flops per token and head, the causal half of the intra-chunk products:
    4 dk dv (state contribution and inter-chunk read-out) + (L + 1)(dk + dv) + 4 dk."""
    dk, dv, L = w.DHQK, w.DHV, w.chunk
    return 4 * dk * dv + (L + 1) * (dk + dv) + 4 * dk


def fwd_work(w: Workload, tensor_path: bool):
    """Algorithmic bytes and flops of one mlstm_fwd, total and per phase.

    The total counts every input read once and every output (h and the final state) written once.
    Per phase, ``bytes`` is what the phase must move of that (inputs it reads, outputs it writes)
    and ``state_traffic`` the chunk- or segment-state bytes the path itself writes and reads
    between its phases (per-segment states on the tensor-core path, per-chunk states on the
    CUDA-core path), which are not algorithmic.  The outputs phase (the walk on the tensor-core
    path) moves exactly bytes_per_token_head per token and head.
    """
    e = 4 if w.dtype == "f32" else 2
    tok = w.B * w.NH * w.S
    dk, dv, L = w.DHQK, w.DHV, w.chunk
    heads = w.B * w.NH
    NC = math.ceil(w.S / L)
    nstate = segments(w) if tensor_path else NC
    state = heads * nstate * 4 * (dk * dv + dk)
    final = heads * 4 * (dk * dv + dk + 1)
    phases = {
        "gate_prep": {"bytes": tok * 8, "state_traffic": tok * 8 + heads * NC * 16, "flops": tok * 10},
        "state_contributions": {"bytes": tok * (e * (dk + dv) + 4), "state_traffic": state,
                                "flops": tok * 2 * dk * (dv + 1)},
        "state_scan": {"bytes": final, "state_traffic": 2 * state, "flops": heads * nstate * 3 * (dk * dv + dk)},
        "outputs": {"bytes": tok * bytes_per_token_head(w), "state_traffic": state,
                    "flops": tok * (2 * dk * dv + (L + 1) * (dk + dv) + 2 * dk)
                    + (tok * 2 * dk * dv if tensor_path else 0)},
    }
    return {"bytes": tok * bytes_per_token_head(w) + final, "flops": tok * flops_per_token_head(w),
            "phases": phases}


def step_work(B, NH, dk, dv, e=2, ogate=True):
    """One mlstm_step: the fp32 state read and written once plus the token I/O."""
    heads = B * NH
    state = heads * 4 * (dk * dv + dk + 1)
    io = heads * (e * (2 * dk + dv + (dv if ogate else 0)) + 8 + e * dv)
    return {"bytes": 2 * state + io, "flops": heads * (6 * dk * dv + 6 * dk)}


def roofline(work: dict, dur_s: float, peaks: dict, tensor: bool):
    """The roofline object of one kernel: its algorithmic bytes (and flops) per launch over its
    measured duration, against the measured HBM copy bandwidth, or the bf16 tensor peak when the
    flops take longer at peak than the bytes."""
    bw, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    fp32_peak = N_SM * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    comp_peak = tc if tensor else fp32_peak
    t_mem = work["bytes"] / (bw * 1e9)
    t_comp = work["flops"] / (comp_peak * 1e12)
    if t_mem >= t_comp:
        r = {"bound": "hbm", "achieved": work["bytes"] / dur_s / 1e9, "peak": bw, "unit": "GB/s"}
    else:
        r = {"bound": "tensor" if tensor else "alu", "achieved": work["flops"] / dur_s / 1e12, "peak": comp_peak,
             "unit": "TFLOP/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["peak_source"] = ("%s (%s)" % (peaks["source"], "of measured" if peaks["source"] == "measured" else
                                     "of fallback")) if r["bound"] != "alu" else \
        "derived: 148 SMs x 128 FP32 lanes x 2 x max clock"
    # the same kernel against the other ceiling, for context
    r["tflops"] = work["flops"] / dur_s / 1e12
    r["frac_tc_peak"] = r["tflops"] / tc if tensor else None
    r["gbs"] = work["bytes"] / dur_s / 1e9
    r["frac_hbm"] = r["gbs"] / bw
    return r


# ---------------------------------------------------------------- clocks

THROTTLE_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons while it runs.

    Through NVML every ``period_s`` (2 ms by default, so that even a timed region of tens of
    milliseconds holds samples), else through ``nvidia-smi -lms 100``.  Only reads: no setting
    of the GPU is changed.
    """

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (time, sm_mhz, sm_max_mhz, set of active reasons)
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        idx = self.cuda_index
        try:
            idx = torch.cuda._get_nvml_device_index(self.cuda_index)
        except Exception:   # noqa: BLE001 - fall back to the CUDA index
            pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def loop():
                while not self._stop.is_set():
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        r = int(get_reasons(h))
                        self.samples.append((time.time(), mhz, sm_max, {n for n, b in bits.items() if r & b}))
                    except Exception:   # noqa: BLE001 - a failed read is skipped
                        pass
                    time.sleep(self.period)
            self.source = "nvml, %.0f ms period" % (self.period * 1e3)
            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            return
        except Exception:   # noqa: BLE001 - no NVML: use nvidia-smi
            pass
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self._proc = subprocess.Popen(["nvidia-smi", "-i", str(self.cuda_index), "--query-gpu=" + q,
                                           "--format=csv,noheader,nounits", "-lms", "100"],
                                          stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.source = "nvidia-smi, 100 ms period"

        def read():
            for line in self._proc.stdout:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 6:
                    try:
                        act = {THROTTLE_NAMES[i] for i in range(4) if parts[2 + i].lower().startswith("active")}
                        self.samples.append((time.time(), float(parts[0]), float(parts[1]), act))
                    except ValueError:
                        pass
        self._thread = threading.Thread(target=read, daemon=True)
        self._thread.start()

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        rows = [r for r in self.samples if t0 <= r[0] <= t1]
        window = "timed region (%.3f s)" % (t1 - t0)
        if len(rows) < 3:
            rows = list(self.samples)
            window = "whole run (fewer than 3 samples inside the %.3f s timed region)" % (t1 - t0)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": rows[0][2],
                "reasons": sorted(set().union(*(r[3] for r in rows))), "samples": len(rows), "window": window,
                "source": self.source}


# ---------------------------------------------------------------- inputs on the device

def device_inputs(w: Workload, nsets: int, device, seed: int):
    """nsets independent forward input sets drawn on the device (timing only; parity lives in tests/)."""
    g = torch.Generator(device=device).manual_seed(seed)
    dt = w.torch_dtype
    sets = []
    for _ in range(nsets):
        shp_qk, shp_v, shp_g = (w.B, w.NH, w.S, w.DHQK), (w.B, w.NH, w.S, w.DHV), (w.B, w.NH, w.S)
        q = (torch.randn(shp_qk, generator=g, device=device) * w.qkv_scale).to(dt)
        k = (torch.randn(shp_qk, generator=g, device=device) * w.qkv_scale).to(dt)
        v = (torch.randn(shp_v, generator=g, device=device) * w.qkv_scale).to(dt)
        i = torch.randn(shp_g, generator=g, device=device) * w.ig[1] + w.ig[0]
        f = torch.randn(shp_g, generator=g, device=device) * w.fg[1] + w.fg[0]
        o = torch.sigmoid(torch.randn(shp_v, generator=g, device=device)).to(dt) if w.ogate else None
        sets.append(dict(q=q, k=k, v=v, i=i, f=f, o=o))
    return sets


def set_bytes(s):
    return sum(t.numel() * t.element_size() for t in s.values() if t is not None)


# ---------------------------------------------------------------- multi-rank host logic

def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time: an all-reduce MAX when a process group is up, else ``ms``."""
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_step_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return world * units_per_step_per_rank * steps / (ms_max / 1e3)


# ---------------------------------------------------------------- our arm

class Runner:
    """Output buffers and workspace of the forward pass of one workload."""

    def __init__(self, w: Workload, device):
        self.w = w
        self.ws = binding.alloc_workspace(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype, device)
        self.h = torch.empty((w.B, w.NH, w.S, w.DHV), dtype=w.torch_dtype, device=device)
        self.C = torch.empty((w.B, w.NH, w.DHQK, w.DHV), dtype=torch.float32, device=device)
        self.n = torch.empty((w.B, w.NH, w.DHQK), dtype=torch.float32, device=device)
        self.m = torch.empty((w.B, w.NH), dtype=torch.float32, device=device)

    def step(self, s, events=None):
        binding.fwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], chunk=self.w.chunk, h_out=self.h,
                    C_final=self.C, n_final=self.n, m_final=self.m, workspace=self.ws, events=events)


def kernel_source_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch of the kernel on the workload, from a committed ncu summary, if its
    kernel source is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get("%s/%s" % (kernel, workload))
        if not e:
            return None
        src = os.path.join(ROOT, e["source"])
        if kernel_source_sha(src) != e["source_sha"]:
            return None
        return e["bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        return None


def workload_for(args) -> Workload:
    """The named workload, with its sequence length (``--seq``) or batch (``--batch``) replaced
    when given (other cases of the same shapes for profiler captures; the JSON line's config shows
    the sizes used)."""
    w = WORKLOADS[args.workload]
    if args.seq:
        w = dataclasses.replace(w, S=args.seq)
    if args.batch:
        w = dataclasses.replace(w, B=args.batch)
    return w


def phase_times(run: Runner, sets, steps: int):
    """Per-phase device time (ms, mean over ``steps`` eager calls), from CUDA events that
    mlstm_fwd_profiled records on the launching stream between its phases."""
    nph = binding.FWD_PHASES
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        run.step(sets[s % len(sets)], events=ev[s])
    torch.cuda.synchronize()
    return {name: sum(ev[s][p].elapsed_time(ev[s][p + 1]) for s in range(steps)) / steps
            for p, name in enumerate(binding.PHASE_NAMES)}


def fwd_report(w: Workload, phase_ms: dict, fwd_ms: float, peaks: dict):
    """Roofline of the dominant kernel (the outputs phase: the walk on the tensor-core path) and the
    whole forward pass against both ceilings."""
    tensor = path_is_tensor(w)
    fw = fwd_work(w, tensor)
    dom = max(binding.PHASE_NAMES, key=lambda k: phase_ms[k])
    wk = fw["phases"][dom]
    uses_tc = tensor and dom in ("state_contributions", "outputs")
    roof = roofline(wk, phase_ms[dom] / 1e3, peaks, uses_tc)
    paired = tensor and binding.fwd_paired_walk(w.DHQK, w.DHV, w.chunk, w.torch_dtype) == 1
    roof["kernel"] = {"outputs": ("walk_pair_kernel" if paired else "walk_kernel") if tensor else "output_simt_kernel",
                      "state_contributions": "segsum_kernel" if tensor else "carry_simt_kernel",
                      "state_scan": "seg_scan_kernel", "gate_prep": "gate kernels"}[dom]
    roof["phase"] = dom
    roof["traffic"] = traffic_for(roof["kernel"], w.name)
    roof["duration_us"] = phase_ms[dom] * 1e3
    roof["algorithmic_bytes"] = wk["bytes"]
    roof["bytes_per_token_head"] = bytes_per_token_head(w) if dom == "outputs" else None
    roof["state_traffic"] = wk["state_traffic"]
    t = fwd_ms / 1e3
    bw, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    fwd = {"ms": fwd_ms, "tflops": fw["flops"] / t / 1e12, "frac_tc_peak": fw["flops"] / t / 1e12 / tc,
           "hbm_gbs": fw["bytes"] / t / 1e9, "frac_hbm": fw["bytes"] / t / 1e9 / bw,
           "frac_roofline": max(fw["flops"] / (tc * 1e12), fw["bytes"] / (bw * 1e9)) / t,
           "algorithmic_bytes": fw["bytes"], "algorithmic_flops": fw["flops"]}
    return roof, fwd


def run_ours(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = workload_for(args)
    peaks = load_peaks()
    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    def barrier():
        if dist:
            torch.distributed.barrier()

    one_set = w.B * w.NH * w.S * ((2 * w.DHQK + 2 * w.DHV) * (4 if w.dtype == "f32" else 2) + 8)
    nsets = max(2, math.ceil(3 * L2_BYTES / max(one_set, 1)))
    nsets = min(nsets, 16)
    if args.sets:
        nsets = max(2, min(nsets, args.sets))
    sets = device_inputs(w, nsets, device, seed=w.seed + 7919 * rank)
    run = Runner(w, device)
    stream = torch.cuda.current_stream()
    nvtx = torch.cuda.nvtx

    # warm-up (eager), also sets kernel attributes before any capture.  NVTX ranges name the
    # bench's parts for a timeline profiler
    nvtx.range_push("bench/warmup")
    for s in range(args.warmup):
        run.step(sets[s % nsets])
    torch.cuda.synchronize()
    nvtx.range_pop()

    # one graph per input set
    graphs = []
    use_graph = not args.no_graph
    if use_graph:
        for s in range(nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run.step(sets[s])
            graphs.append(g)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.05)
    # ---- timed region: exactly K steps
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nvtx.range_push("bench/timed")
    tw0 = time.time()
    ev0.record()
    for s in range(args.steps):
        if use_graph:
            graphs[s % nsets].replay()
        else:
            run.step(sets[s % nsets])
    ev1.record()
    torch.cuda.synchronize()
    tw1 = time.time()
    nvtx.range_pop()
    clocks.stop()
    barrier()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), device)

    # ---- per-phase timing (eager, the same K steps, events on the launching stream)
    nvtx.range_push("bench/phases")
    phase_ms = phase_times(run, sets, args.steps)
    nvtx.range_pop()

    # ---- end to end through the public API with host buffers (pinned), eager.  Every step copies
    # its inputs host -> device and its outputs (h and the final state) back.  Steps are pipelined
    # over three streams: the inputs of step s + 1 go up while step s computes and the outputs of
    # step s - 1 come down; two input buffers and two output sets alternate.
    e2e_steps = min(args.steps, E2E_MAX_STEPS)
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in sets[0].items()}
    devs = [sets[0], sets[1 % nsets]]
    runs = [run, Runner(w, device)]
    outs_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (run.h, run.C, run.n, run.m)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = sum(t.numel() * t.element_size() for t in outs_host)
    s_up, s_comp, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up_done, comp_done, down_done = [None] * e2e_steps, [None] * e2e_steps, [None] * e2e_steps
    nvtx.range_push("bench/e2e")
    e0.record(stream)
    for st in (s_up, s_comp, s_down):
        st.wait_event(e0)
    for s in range(e2e_steps):
        b = s & 1
        if s >= 2:
            s_up.wait_event(comp_done[s - 2])        # the buffer's previous step has read its inputs
        with torch.cuda.stream(s_up):
            for key, hv in host.items():
                if hv is not None:
                    devs[b][key].copy_(hv, non_blocking=True)
        up_done[s] = ev()
        up_done[s].record(s_up)
        s_comp.wait_event(up_done[s])
        if s >= 2:
            s_comp.wait_event(down_done[s - 2])      # the output set's previous results are on the host
        with torch.cuda.stream(s_comp):
            runs[b].step(devs[b])
        comp_done[s] = ev()
        comp_done[s].record(s_comp)
        s_down.wait_event(comp_done[s])
        with torch.cuda.stream(s_down):
            for dst, src in zip(outs_host, (runs[b].h, runs[b].C, runs[b].n, runs[b].m)):
                dst.copy_(src, non_blocking=True)
        down_done[s] = ev()
        down_done[s].record(s_down)
    for st in (s_up, s_comp, s_down):
        stream.wait_stream(st)
    e1.record(stream)
    torch.cuda.synchronize()
    nvtx.range_pop()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    del runs, devs, host, outs_host

    tokens_per_step = w.B * w.S
    value = job_throughput(world, tokens_per_step, args.steps, ms_max)
    e2e_value = job_throughput(world, tokens_per_step, e2e_steps, e2e_ms)

    fwd_ms = sum(phase_ms[k] for k in binding.PHASE_NAMES)
    roof, fwd = fwd_report(w, phase_ms, fwd_ms, peaks)
    graph_fwd = {"ms": ms_max / args.steps}
    fw = fwd_work(w, path_is_tensor(w))
    graph_fwd["tflops"] = fw["flops"] / (graph_fwd["ms"] / 1e3) / 1e12
    graph_fwd["frac_tc_peak"] = graph_fwd["tflops"] / peaks["bf16_tflops"]
    graph_fwd["hbm_gbs"] = fw["bytes"] / (graph_fwd["ms"] / 1e3) / 1e9
    graph_fwd["frac_hbm"] = graph_fwd["hbm_gbs"] / peaks["hbm_gbs"]

    launches_per_step = binding.fwd_kernel_launches(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype)
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded on device; distributions of the workload)",
        "config": {"workload": w.name, "B": w.B, "NH": w.NH, "S": w.S, "DHQK": w.DHQK, "DHV": w.DHV,
                   "chunk": w.chunk, "ogate": w.ogate, "step": "one mlstm_fwd over B x S tokens",
                   "tokens_per_step_per_gpu": tokens_per_step, "parallelism": "replicas x%d" % world,
                   "l2": "%d input sets of %.0f MB each (> L2) in rotation" % (nsets, set_bytes(sets[0]) / 1e6),
                   "timing": "CUDA graph replay" if use_graph else "eager"},
        "roofline": roof,
        "cpu_baseline": None,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "pipeline": "upload, compute and download of consecutive steps on three streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(tw0, tw1),
        "phases_us": {k: round(v * 1e3, 2) for k, v in phase_ms.items()},
        "fwd": graph_fwd,
        "fwd_eager_phases": fwd,
        "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"], "source": peaks["source"]},
    }
    graphs.clear()
    del sets, run
    torch.cuda.empty_cache()
    if args.extras and rank == 0:
        nvtx.range_push("bench/extras")
        out["workloads"] = extras(device, peaks, skip=w.name)
        nvtx.range_pop()
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def path_is_tensor(w: Workload) -> bool:
    """True when the library takes its tensor-core path for this workload."""
    return binding.fwd_tensor_path(w.DHQK, w.DHV, w.chunk, w.torch_dtype) == 1


def fwd_extra(w: Workload, device, peaks, reps: int = 20):
    """One forward workload timed alone: eager calls between events, then per-phase events; the
    roofline of its dominant kernel and the whole pass against both ceilings."""
    sets = device_inputs(w, 2, device, seed=w.seed)
    run = Runner(w, device)
    for s in range(3):
        run.step(sets[s % 2])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(reps):
        run.step(sets[s % 2])
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / reps / 1e3
    phase_ms = phase_times(run, sets, reps)
    roof, fwd = fwd_report(w, phase_ms, t * 1e3, peaks)
    del sets, run
    torch.cuda.empty_cache()
    return {"ms": t * 1e3, "tokens_per_s": w.B * w.S / t, "tflops": fwd["tflops"], "frac_tc_peak": fwd["frac_tc_peak"],
            "hbm_gbs": fwd["hbm_gbs"], "frac_roofline": fwd["frac_roofline"], "roofline": roof,
            "phases_us": {k: round(v * 1e3, 2) for k, v in phase_ms.items()},
            "l2": "2 input sets of %.0f MB in rotation" % (w.B * w.NH * w.S * bytes_per_token_head(w) / 1e6)}


def step_extra(device, peaks, nsteps: int = 200):
    """The decode step on its workload (B256 NH8 d256/512, a 1 GiB fp32 state, larger than L2)."""
    w = WORKLOADS["step_bf16"]
    C = torch.randn((w.B, w.NH, w.DHQK, w.DHV), device=device) * 0.01
    n = torch.randn((w.B, w.NH, w.DHQK), device=device) * 0.01
    m = torch.zeros((w.B, w.NH), device=device)
    g = torch.Generator(device=device).manual_seed(5)
    toks = []
    for _ in range(4):
        r = lambda *shape: torch.randn(shape, generator=g, device=device)
        toks.append({"q": r(w.B, w.NH, w.DHQK).to(torch.bfloat16), "k": r(w.B, w.NH, w.DHQK).to(torch.bfloat16),
                     "v": r(w.B, w.NH, w.DHV).to(torch.bfloat16), "i": r(w.B, w.NH) * w.ig[1] + w.ig[0],
                     "f": r(w.B, w.NH) * w.fg[1] + w.fg[0],
                     "o": torch.sigmoid(r(w.B, w.NH, w.DHV)).to(torch.bfloat16)})
    hd = torch.empty((w.B, w.NH, w.DHV), dtype=torch.bfloat16, device=device)
    for t in toks:
        binding.step(C, n, m, t["q"], t["k"], t["v"], t["i"], t["f"], t["o"], h_out=hd)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(nsteps):
        t = toks[s % 4]
        binding.step(C, n, m, t["q"], t["k"], t["v"], t["i"], t["f"], t["o"], h_out=hd)
    e1.record()
    torch.cuda.synchronize()
    ts = e0.elapsed_time(e1) / nsteps / 1e3
    sw = step_work(w.B, w.NH, w.DHQK, w.DHV)
    roof = roofline(sw, ts, peaks, False)
    roof["kernel"] = "step_kernel"
    roof["traffic"] = traffic_for("step_kernel", w.name)
    roof["duration_us"] = ts * 1e6
    return {"workload": "B%d NH%d d%d/%d, fp32 state (1 GiB)" % (w.B, w.NH, w.DHQK, w.DHV),
            "us_per_step": ts * 1e6, "gbs": sw["bytes"] / ts / 1e9, "frac_hbm": sw["bytes"] / ts / 1e9 / peaks["hbm_gbs"],
            "steps": nsteps, "roofline": roof}


def bwd_work(w: Workload):
    """Algorithmic work of one mlstm_bwd: per token and head the products of the chunkwise gradient
    (the forward read-out recomputed, 2 dk dv; the chunk-start states recomputed, 2 dk dv; the
    read-out's state gradient and the dq, dk, dv inter-chunk terms, 4 x 2 dk dv; the causal half of
    the intra-chunk products, 3 (L + 1)(dk + dv)), i.e. 14 dk dv + 3 (L + 1)(dk + dv) flops; bytes:
    q, k, v, o, dh and both gates read once, dq, dk, dv, do and both gate gradients written once."""
    e = 4 if w.dtype == "f32" else 2
    tok = w.B * w.NH * w.S
    dk, dv, L = w.DHQK, w.DHV, w.chunk
    flops = tok * (14 * dk * dv + 3 * (L + 1) * (dk + dv))
    io = e * (2 * dk + dv) + (e * dv if w.ogate else 0) + e * dv + 8
    out = e * (2 * dk + dv) + (e * dv if w.ogate else 0) + 8
    return {"flops": flops, "bytes": tok * (io + out)}


def bwd_extra(w: Workload, device, peaks, reps: int = 5):
    """The backward pass on a forward workload's shape (dh ~ N(0, 1)), timed alone with events."""
    s = device_inputs(w, 1, device, seed=w.seed)[0]
    g = torch.Generator(device=device).manual_seed(w.seed + 1)
    dh = torch.randn((w.B, w.NH, w.S, w.DHV), generator=g, device=device).to(w.torch_dtype)
    ws = torch.empty(binding.bwd_workspace_size(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype),
                     dtype=torch.uint8, device=device)
    out = (torch.empty_like(s["q"]), torch.empty_like(s["k"]), torch.empty_like(s["v"]), torch.empty_like(s["i"]),
           torch.empty_like(s["f"]), None if s["o"] is None else torch.empty_like(s["o"]))
    call = lambda: binding.bwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], dh, chunk=w.chunk, workspace=ws, out=out)
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / reps / 1e3
    bw = bwd_work(w)
    tensor = binding.bwd_tensor_path(w.DHQK, w.DHV, w.chunk, w.torch_dtype) == 1
    roof = roofline(bw, t, peaks, tensor)
    roof["kernel"] = "mlstm_bwd (all kernels of the call)"
    del s, dh, ws, out
    torch.cuda.empty_cache()
    return {"workload": "%s shape (B%d NH%d S%d d%d/%d chunk %d, %s)" % (w.name, w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk,
                                                                        w.dtype),
            "ms": t * 1e3, "tokens_per_s": w.B * w.S / t, "tflops": bw["flops"] / t / 1e12,
            "products": ("read-out numerator, its state gradient and dq, dk, dv on tcgen05 (bf16 operands, fp32 "
                         "accumulation); scores, dS and the scans on the CUDA cores") if tensor else
                        "every product on the CUDA cores (fp32)",
            "kernel_launches": "gate preprocessing, chunk-start states, scores, numerator, dS, state gradient, "
                               "state-gradient scan, dq, dk, dv, gate gradients", "roofline": roof}


def extras(device, peaks, skip=None):
    """Per-workload numbers for the other shapes (eager, events)."""
    res = {}
    for name in ("fwd_bf16_d256", "fwd_bf16_7b", "fwd_bf16_long"):
        if name != skip:
            res[name] = fwd_extra(WORKLOADS[name], device, peaks)
    res["step_bf16"] = step_extra(device, peaks)
    res["bwd_bf16_7b"] = bwd_extra(WORKLOADS["fwd_bf16_7b"], device, peaks)
    res["slstm_f32"] = slstm_extra(device, peaks)
    return res


def slstm_work(B, S, NH, DH, esize):
    """Algorithmic work of one slstm_fwd call: the recurrent products (2 x 4 DH^2 flops per cell
    group and step) and the bytes of wx read and h written once."""
    return {"flops": 2.0 * 4 * DH * DH * NH * B * S, "bytes": (4 + 1) * NH * DH * B * S * esize}


def slstm_extra(device, peaks, B=None, S=None):
    """The sLSTM recurrence on its workload: one slstm_fwd call over the whole sequence (batch
    and sequence length overridable for profiling)."""
    from xlstm_mlstm_cell_b200.workloads import SLSTM_WORKLOADS, make_slstm_inputs
    w = SLSTM_WORKLOADS["slstm_f32"]
    w = dataclasses.replace(w, B=B or w.B, S=S or w.S)
    wx, R = make_slstm_inputs(w.B, w.S, w.NH, w.DH, w.dtype, w.seed, w.f_loc)
    wx, R = wx.to(device), R.to(device)
    h_out = torch.empty((w.B, w.S, w.NH, w.DH), dtype=wx.dtype, device=device)
    state = tuple(torch.zeros((w.B, w.NH, w.DH), device=device) for _ in range(4))
    for _ in range(2):
        for x in state:
            x.zero_()
        binding.slstm_fwd(wx, R, forget=w.forget, state=state, h_out=h_out)
    torch.cuda.synchronize()
    reps = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        binding.slstm_fwd(wx, R, forget=w.forget, state=state, h_out=h_out)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / reps / 1e3
    sw = slstm_work(w.B, w.S, w.NH, w.DH, wx.element_size())
    fp32_peak = N_SM * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    return {"workload": "B%d S%d NH%d DH%d %s, %s forget gate" % (w.B, w.S, w.NH, w.DH, w.dtype, w.forget),
            "ms": t * 1e3, "tokens_per_s": w.B * w.S / t, "us_per_step": t / w.S * 1e6,
            "tflops": sw["flops"] / t / 1e12, "bound": "alu", "frac_fp32_peak": sw["flops"] / t / 1e12 / fp32_peak,
            "fp32_peak_tflops": fp32_peak, "hbm_gbs": sw["bytes"] / t / 1e9,
            "batch_per_cluster": binding.slstm_batch_per_cluster(w.B, w.NH, w.DH, wx.dtype)}


# ---------------------------------------------------------------- the oracle as CPU baseline / reference arm

def oracle_inputs(w: Workload, tokens: int):
    """The first ``tokens`` tokens of every head of the workload's seeded inputs (CPU)."""
    from xlstm_mlstm_cell_b200.workloads import make_fwd_inputs
    return make_fwd_inputs(w, S=min(tokens, w.S))


def oracle_time(inputs, threads):
    import oracle
    t0 = time.perf_counter()
    oracle.mlstm_fwd(*inputs, nthreads=threads)
    return time.perf_counter() - t0


def cpu_baseline(w: Workload, target_s: float = 12.0):
    """The fp64 oracle, as it stands, on the host cores: a bounded sample of the workload (every
    batch element and head, the first S' tokens, S' sized so that the run takes about
    ``target_s``), reported in the bench's unit (tokens/s)."""
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    probe = min(w.S, 1024)
    t_probe = oracle_time(oracle_inputs(w, probe), threads)
    tokens = int(min(w.S, max(probe, probe * target_s / max(t_probe, 1e-3))))
    tokens = max(probe, tokens // 64 * 64) if tokens < w.S else w.S
    t = oracle_time(oracle_inputs(w, tokens), threads)
    return {"value": w.B * tokens / t, "unit": "tokens/s", "cores": min(threads, w.B * w.NH), "kind": "oracle",
            "sample": "mlstm_fwd over the first %d of %d tokens, all B=%d x NH=%d heads, %.1f s wall "
                      "(a thread per head, %d host cores)" % (tokens, w.S, w.B, w.NH, t, threads)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload_for(args)
    import oracle
    oracle.build()
    threads = oracle.default_threads()
    tokens = min(w.S, REF_SAMPLE_TOKENS)
    inputs = oracle_inputs(w, tokens)
    for _ in range(args.warmup):
        oracle_time(inputs, threads)
    dt = sum(oracle_time(inputs, threads) for _ in range(args.steps))
    value = args.steps * w.B * tokens / dt
    cores = min(threads, w.B * w.NH)
    sample = "each step: mlstm_fwd over the first %d of %d tokens, all B=%d x NH=%d heads" % (tokens, w.S, w.B, w.NH)
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, CPU)",
           "config": {"workload": w.name, "B": w.B, "NH": w.NH, "S": w.S, "DHQK": w.DHQK, "DHV": w.DHV,
                      "chunk": w.chunk, "ogate": w.ogate, "sample_tokens_per_head": tokens},
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=[k for k in WORKLOADS if k.startswith("fwd_")])
    ap.add_argument("--extras", type=int, default=1, help="also time the other workloads (rank 0)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq", type=int, default=0, help="override the workload's sequence length (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size (profiling)")
    ap.add_argument("--sets", type=int, default=0, help="cap the number of rotated input sets (profiling)")
    ap.add_argument("--slstm", action="store_true",
                    help="time only the sLSTM recurrence workload (sizes from --batch / --seq) and print its numbers")
    ap.add_argument("--decode", action="store_true", help="time only the decode step workload and print its numbers")
    ap.add_argument("--bwd", action="store_true",
                    help="time only the backward pass on the workload's shape (sizes from --batch / --seq)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    binding.load()
    if args.bwd:
        torch.cuda.set_device(local_rank)
        print(json.dumps(bwd_extra(workload_for(args), torch.device("cuda", local_rank), load_peaks())))
        return
    if args.slstm or args.decode:
        torch.cuda.set_device(local_rank)
        dev = torch.device("cuda", local_rank)
        res = slstm_extra(dev, load_peaks(), B=args.batch or None, S=args.seq or None) if args.slstm else \
            step_extra(dev, load_peaks(), nsteps=max(args.steps, 1))
        print(json.dumps(res))
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
