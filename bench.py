#!/usr/bin/env python
"""Benchmark of libmlstm on B200: one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic input:
``mlstm_fwd`` over the workload's B x S prefill tokens (gate preprocessing,
chunk-state carry, chunk outputs) followed by one ``mlstm_step`` decode token on
the state it returns.  ``value`` is tokens per second over the whole job
(B x (S + 1) tokens per step per GPU), timed with CUDA events around exactly
``--steps`` graph replays, the max over ranks.  Inputs live in HBM before the
timed region; several input sets, together larger than the 126 MB L2, are used
in rotation so that no step reads its inputs from L2.

Heads and batches are independent, so N GPUs run N independent replicas of the
workload with no collective ("weak" scaling); the only collectives are the
barrier and the max of the timings.

``--impl reference`` times the fp64 CPU oracle (the plain recurrence) on the
same workload instead, on rank 0 only.
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
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
FP32_LANES_PER_SM, N_SM = 128, 148


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


def fwd_work(w: Workload, tensor_path: bool):
    """Algorithmic bytes and flops of one mlstm_fwd, total and per phase.

    Bytes count every input read once and every output written once; flops
    count the causal half of the intra-chunk products (masked work excluded).
    Per token and head: 4 dk dv (state contribution and inter-chunk read-out)
    + (L + 1)(dk + dv) (intra-chunk) + 4 dk.  Per phase, the state traffic is
    the path's own: per-segment states on the tensor-core path, per-chunk
    states on the CUDA-core path.
    """
    e = 4 if w.dtype == "f32" else 2
    tok = w.B * w.NH * w.S
    dk, dv, L = w.DHQK, w.DHV, w.chunk
    heads = w.B * w.NH
    NC = math.ceil(w.S / L)
    nstate = segments(w) if tensor_path else NC
    state = heads * nstate * 4 * (dk * dv + dk)
    in_bytes = tok * (e * (2 * dk + dv) + (e * dv if w.ogate else 0) + 8)
    out_bytes = tok * e * dv + heads * 4 * (dk * dv + dk + 1)
    flops_tok = 4 * dk * dv + (L + 1) * (dk + dv) + 4 * dk
    phases = {
        "gate_prep": {"bytes": tok * 16 + heads * NC * 16, "flops": tok * 10},
        "state_contributions": {"bytes": tok * (e * (dk + dv) + 12) + state, "flops": tok * 2 * dk * (dv + 1)},
        "state_scan": {"bytes": 2 * state, "flops": heads * nstate * 3 * (dk * dv + dk)},
        "outputs": {"bytes": tok * (e * (2 * dk + dv) + (e * dv if w.ogate else 0) + e * dv + 12) + state,
                    "flops": tok * (2 * dk * dv + (L + 1) * (dk + dv) + 2 * dk)
                    + (tok * 2 * dk * dv if tensor_path else 0)},
    }
    return {"bytes": in_bytes + out_bytes, "flops": tok * flops_tok, "phases": phases}


def step_work(B, NH, dk, dv, e=2, ogate=True):
    """One mlstm_step: the fp32 state read and written once plus the token I/O."""
    heads = B * NH
    state = heads * 4 * (dk * dv + dk + 1)
    io = heads * (e * (2 * dk + dv + (dv if ogate else 0)) + 8 + e * dv)
    return {"bytes": 2 * state + io, "flops": heads * (6 * dk * dv + 6 * dk)}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while it runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [p for (t, p) in self.samples if t0 <= t <= t1]
        window = "timed region"
        if len(rows) < 3:   # a timed region shorter than the sampling period: use the whole run
            rows = [p for (_, p) in self.samples]
            window = "whole run (timed region shorter than the sampling period)"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "window": window}


# ---------------------------------------------------------------- inputs on the device

def device_inputs(w: Workload, nsets: int, device, seed: int):
    """nsets independent input sets drawn on the device (timing only; parity lives in tests/)."""
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
        tq = torch.randn((w.B, w.NH, w.DHQK), generator=g, device=device).to(dt)
        tk = torch.randn((w.B, w.NH, w.DHQK), generator=g, device=device).to(dt)
        tv = torch.randn((w.B, w.NH, w.DHV), generator=g, device=device).to(dt)
        ti = torch.randn((w.B, w.NH), generator=g, device=device) * w.ig[1] + w.ig[0]
        tf = torch.randn((w.B, w.NH), generator=g, device=device) * w.fg[1] + w.fg[0]
        to = torch.sigmoid(torch.randn((w.B, w.NH, w.DHV), generator=g, device=device)).to(dt) if w.ogate else None
        sets.append(dict(q=q, k=k, v=v, i=i, f=f, o=o, tq=tq, tk=tk, tv=tv, ti=ti, tf=tf, to=to))
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
    """Buffers and the two library calls of one step."""

    def __init__(self, w: Workload, device):
        self.w = w
        self.ws = binding.alloc_workspace(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype, device)
        self.h = torch.empty((w.B, w.NH, w.S, w.DHV), dtype=w.torch_dtype, device=device)
        self.C = torch.empty((w.B, w.NH, w.DHQK, w.DHV), dtype=torch.float32, device=device)
        self.n = torch.empty((w.B, w.NH, w.DHQK), dtype=torch.float32, device=device)
        self.m = torch.empty((w.B, w.NH), dtype=torch.float32, device=device)
        self.hd = torch.empty((w.B, w.NH, w.DHV), dtype=w.torch_dtype, device=device)

    def step(self, s, events=None, step_events=None):
        binding.fwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], chunk=self.w.chunk, h_out=self.h,
                    C_final=self.C, n_final=self.n, m_final=self.m, workspace=self.ws, events=events)
        if step_events:
            step_events[0].record()
        binding.step(self.C, self.n, self.m, s["tq"], s["tk"], s["tv"], s["ti"], s["tf"], s["to"], h_out=self.hd)
        if step_events:
            step_events[1].record()


def kernel_source_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def traffic_for(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if its kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(kernel)
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

    # warm-up (eager), also sets kernel attributes before any capture.  NVTX ranges name the
    # bench's parts for a timeline profiler
    nvtx = torch.cuda.nvtx
    nvtx.range_push("bench/warmup")
    for s in range(args.warmup):
        run.step(sets[s % nsets])
    torch.cuda.synchronize()
    nvtx.range_pop()

    # capture one graph per input set
    graphs = []
    use_graph = not args.no_graph
    if use_graph:
        for s in range(nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run.step(sets[s])
            graphs.append(g)
        for g in graphs[:2]:
            g.replay()
        torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
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
    barrier()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), device)

    # ---- per-phase timing (eager, the same K steps, events on the launching stream)
    nph = binding.FWD_PHASES
    ph_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(args.steps)]
    st_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    nvtx.range_push("bench/phases")
    tp0 = time.time()
    for s in range(args.steps):
        run.step(sets[s % nsets], events=ph_ev[s], step_events=st_ev[s])
    torch.cuda.synchronize()
    tp1 = time.time()
    nvtx.range_pop()
    phase_ms = {name: sum(ph_ev[s][p].elapsed_time(ph_ev[s][p + 1]) for s in range(args.steps)) / args.steps
                for p, name in enumerate(binding.PHASE_NAMES)}
    phase_ms["decode_step"] = sum(st_ev[s][0].elapsed_time(st_ev[s][1]) for s in range(args.steps)) / args.steps

    # ---- end to end through the public API with host buffers (pinned), eager.  Every step copies
    # its inputs host -> device and its outputs (h of the prefill and of the decode step) back.
    # Steps are pipelined over three streams: the inputs of step s + 1 go up while step s computes
    # and the outputs of step s - 1 come down; two input buffers and two output sets alternate.
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in sets[0].items()}
    devs = [sets[0], sets[1 % nsets]]
    runs = [run, Runner(w, device)]
    h_host = torch.empty(run.h.shape, dtype=run.h.dtype).pin_memory()
    hd_host = torch.empty(run.hd.shape, dtype=run.hd.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = h_host.numel() * h_host.element_size() + hd_host.numel() * hd_host.element_size()
    s_up, s_comp, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up_done, comp_done, down_done = [None] * args.steps, [None] * args.steps, [None] * args.steps
    nvtx.range_push("bench/e2e")
    te0 = time.time()
    e0.record(stream)
    for st in (s_up, s_comp, s_down):
        st.wait_event(e0)
    for s in range(args.steps):
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
            h_host.copy_(runs[b].h, non_blocking=True)
            hd_host.copy_(runs[b].hd, non_blocking=True)
        down_done[s] = ev()
        down_done[s].record(s_down)
    for st in (s_up, s_comp, s_down):
        stream.wait_stream(st)
    e1.record(stream)
    torch.cuda.synchronize()
    te1 = time.time()
    nvtx.range_pop()
    clocks.stop()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)

    tokens_per_step = w.B * (w.S + 1)
    value = job_throughput(world, tokens_per_step, args.steps, ms_max)
    e2e_value = job_throughput(world, tokens_per_step, args.steps, e2e_ms)

    # ---- roofline of the dominant kernel
    fw = fwd_work(w, path_is_tensor(w))
    sw = step_work(w.B, w.NH, w.DHQK, w.DHV, 4 if w.dtype == "f32" else 2, w.ogate)
    works = dict(fw["phases"])
    works["decode_step"] = sw
    dom = max((k for k in works if k in phase_ms), key=lambda k: phase_ms[k])
    dur_s = phase_ms[dom] / 1e3
    bw = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops"]
    fp32_peak = N_SM * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    wk = works[dom]
    uses_tc = w.dtype == "bf16" and dom in ("state_contributions", "outputs") and path_is_tensor(w)
    comp_peak = tc if uses_tc else fp32_peak
    t_mem = wk["bytes"] / (bw * 1e9)
    t_comp = wk["flops"] / (comp_peak * 1e12)
    if t_mem >= t_comp:
        roof = {"bound": "hbm", "achieved": wk["bytes"] / dur_s / 1e9, "peak": bw, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor" if uses_tc else "alu", "achieved": wk["flops"] / dur_s / 1e12, "peak": comp_peak,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"] if roof["bound"] != "alu" else "derived: 148 SMs x 128 FP32 lanes x 2 x max clock"
    roof["traffic"] = traffic_for(dom)
    roof["duration_us"] = phase_ms[dom] * 1e3

    launches_per_step = binding.fwd_kernel_launches(w.B, w.NH, w.S, w.DHQK, w.DHV, w.chunk, w.torch_dtype) + 1
    fwd_ms = sum(phase_ms[k] for k in binding.PHASE_NAMES)
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
                   "chunk": w.chunk, "ogate": w.ogate, "step": "mlstm_fwd over B x S + one mlstm_step",
                   "tokens_per_step_per_gpu": tokens_per_step, "parallelism": "replicas x%d" % world,
                   "l2": "%d input sets (%.0f MB) in rotation > L2" % (nsets, nsets * set_bytes(sets[0]) / 1e6),
                   "timing": "CUDA graph replay" if use_graph else "eager"},
        "roofline": roof,
        "cpu_baseline": None,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipeline": "upload, compute and download of consecutive steps on three streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(tw0, tw1),
        "phases_us": {k: round(v * 1e3, 2) for k, v in phase_ms.items()},
        "fwd": {"tflops": fw["flops"] / (fwd_ms / 1e3) / 1e12,
                "frac_tc_peak": fw["flops"] / (fwd_ms / 1e3) / 1e12 / tc,
                "hbm_gbs": fw["bytes"] / (fwd_ms / 1e3) / 1e9,
                "frac_roofline": max(fw["flops"] / (tc * 1e12), fw["bytes"] / (bw * 1e9)) / (fwd_ms / 1e3)},
        "decode_step": {"gbs": sw["bytes"] / (phase_ms["decode_step"] / 1e3) / 1e9,
                        "frac_hbm": sw["bytes"] / (phase_ms["decode_step"] / 1e3) / 1e9 / bw},
        "peaks": {"hbm_gbs": bw, "bf16_tflops": tc, "source": peaks["source"]},
    }
    if args.extras and rank == 0:
        nvtx.range_push("bench/extras")
        out["workloads"] = extras(device, peaks)
        nvtx.range_pop()
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    graphs.clear()
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def path_is_tensor(w: Workload) -> bool:
    """True when the library takes its tensor-core path for this workload."""
    return binding.fwd_tensor_path(w.DHQK, w.DHV, w.chunk, w.torch_dtype) == 1


def extras(device, peaks):
    """Per-workload numbers for the other shapes (timing only, eager, events)."""
    res = {}
    bw, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    for name in ("fwd_bf16_7b", "fwd_bf16_long"):
        w = WORKLOADS[name]
        s = device_inputs(w, 1, device, seed=w.seed)[0]
        run = Runner(w, device)
        for _ in range(2):
            binding.fwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], chunk=w.chunk, h_out=run.h,
                        C_final=run.C, n_final=run.n, m_final=run.m, workspace=run.ws)
        torch.cuda.synchronize()
        reps = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            binding.fwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], chunk=w.chunk, h_out=run.h,
                        C_final=run.C, n_final=run.n, m_final=run.m, workspace=run.ws)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / reps / 1e3
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(binding.FWD_PHASES + 1)]
        binding.fwd(s["q"], s["k"], s["v"], s["i"], s["f"], s["o"], chunk=w.chunk, h_out=run.h, C_final=run.C,
                    n_final=run.n, m_final=run.m, workspace=run.ws, events=ev)
        torch.cuda.synchronize()
        phases = {nm: round(ev[p].elapsed_time(ev[p + 1]) * 1e3, 1) for p, nm in enumerate(binding.PHASE_NAMES)}
        fw = fwd_work(w, path_is_tensor(w))
        res[name] = {"ms": t * 1e3, "tokens_per_s": w.B * w.S / t, "tflops": fw["flops"] / t / 1e12,
                     "frac_tc_peak": fw["flops"] / t / 1e12 / tc, "hbm_gbs": fw["bytes"] / t / 1e9,
                     "frac_roofline": max(fw["flops"] / (tc * 1e12), fw["bytes"] / (bw * 1e9)) / t,
                     "phases_us": phases}
        del s, run
        torch.cuda.empty_cache()
    w = WORKLOADS["step_bf16"]
    C = torch.randn((w.B, w.NH, w.DHQK, w.DHV), device=device) * 0.01
    n = torch.randn((w.B, w.NH, w.DHQK), device=device) * 0.01
    m = torch.zeros((w.B, w.NH), device=device)
    toks = device_inputs(Workload("tok", "bf16", w.B, w.NH, 1, w.DHQK, w.DHV, 16, 1.0, w.ig, w.fg, True, 5), 4,
                         device, seed=5)
    hd = torch.empty((w.B, w.NH, w.DHV), dtype=torch.bfloat16, device=device)
    sq = lambda x: x[:, :, 0].contiguous()
    toks = [{k: sq(v) for k, v in t.items() if k in ("q", "k", "v", "i", "f", "o")} for t in toks]
    for t in toks:
        binding.step(C, n, m, t["q"], t["k"], t["v"], t["i"], t["f"], t["o"], h_out=hd)
    torch.cuda.synchronize()
    nsteps = 200
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(nsteps):
        t = toks[s % 4]
        binding.step(C, n, m, t["q"], t["k"], t["v"], t["i"], t["f"], t["o"], h_out=hd)
    e1.record()
    torch.cuda.synchronize()
    ts = e0.elapsed_time(e1) / nsteps / 1e3
    sw = step_work(w.B, w.NH, w.DHQK, w.DHV)
    res["step_bf16"] = {"us_per_step": ts * 1e6, "gbs": sw["bytes"] / ts / 1e9, "frac_hbm": sw["bytes"] / ts / 1e9 / bw,
                        "steps": nsteps}
    res["slstm_f32"] = slstm_extra(device, peaks)
    return res


def slstm_work(B, S, NH, DH, esize):
    """Algorithmic work of one slstm_fwd call: the recurrent products (2 x 4 DH^2 flops per cell
    group and step) and the bytes of wx read and h written once."""
    return {"flops": 2.0 * 4 * DH * DH * NH * B * S, "bytes": (4 + 1) * NH * DH * B * S * esize}


def slstm_extra(device, peaks, B=None, S=None):
    """The sLSTM recurrence on its workload: one slstm_fwd call over the whole sequence (batch
    and sequence length overridable for profiling)."""
    import dataclasses
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

def oracle_sample(w: Workload, target_s: float = 10.0, max_reps: int = 20):
    """Times the fp64 oracle on the workload's first batch element(s): fwd over S tokens + one step."""
    import oracle
    from xlstm_mlstm_cell_b200.workloads import make_fwd_inputs
    Bs = 1
    inputs = make_fwd_inputs(w, B=Bs)
    tok = [x[:, :, :1] if x is not None else None for x in inputs]
    threads = oracle.default_threads()
    oracle.build()
    reps, t_total = 0, 0.0
    while reps < max_reps and (t_total < target_s or reps == 0):
        t0 = time.perf_counter()
        h, C, n, m = oracle.mlstm_fwd(*inputs, nthreads=threads)
        oracle.mlstm_step(C, n, m, *(x[:, :, 0] if x is not None else None for x in tok), nthreads=threads)
        t_total += time.perf_counter() - t0
        reps += 1
    tokens = reps * Bs * (w.S + 1)
    return {"value": tokens / t_total, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d x (B=%d of %d, NH=%d, S=%d fwd + 1 step), %.1f s wall" % (reps, Bs, w.B, w.NH, w.S,
                                                                                   t_total)}


def cpu_baseline(w: Workload):
    return oracle_sample(w)


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload_for(args)
    import oracle
    from xlstm_mlstm_cell_b200.workloads import make_fwd_inputs
    oracle.build()
    threads = oracle.default_threads()
    Bs = 1
    inputs = make_fwd_inputs(w, B=Bs)

    def one():
        h, C, n, m = oracle.mlstm_fwd(*inputs, nthreads=threads)
        oracle.mlstm_step(C, n, m, *(x[:, :, 0] if x is not None else None for x in inputs), nthreads=threads)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    value = args.steps * Bs * (w.S + 1) / dt
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, CPU)",
           "config": {"workload": w.name, "B": w.B, "NH": w.NH, "S": w.S, "DHQK": w.DHQK, "DHV": w.DHV,
                      "chunk": w.chunk, "sample_B": Bs},
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": "B=%d of %d per step (fwd over S + 1 step)" % (Bs, w.B)},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fwd_bf16_d256", choices=[k for k in WORKLOADS if k.startswith("fwd_")])
    ap.add_argument("--extras", type=int, default=1, help="also time the other workloads (rank 0)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq", type=int, default=0, help="override the workload's sequence length (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size (profiling)")
    ap.add_argument("--sets", type=int, default=0, help="cap the number of rotated input sets (profiling)")
    ap.add_argument("--slstm", action="store_true",
                    help="time only the sLSTM recurrence workload (sizes from --batch / --seq) and print its numbers")
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
    if args.slstm:
        torch.cuda.set_device(local_rank)
        print(json.dumps(slstm_extra(torch.device("cuda", local_rank), load_peaks(), B=args.batch or None,
                                     S=args.seq or None)))
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
