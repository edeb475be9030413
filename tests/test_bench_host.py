"""Host-side arithmetic of the benchmark (no GPU): the algorithmic work that the roofline fractions
divide by, and the workload overrides used by profiler captures."""
from __future__ import annotations

import argparse
import dataclasses

import bench
from xlstm_mlstm_cell_b200.workloads import WORKLOADS


def test_walk_bytes_per_token_and_head():
    # the per-token figure of the algorithmic bytes: q, k, v (and o) read, h written, two gate
    # pre-activations read: 2 (2 dk + dv) + 2 dv [o] + 2 dv + 8
    assert bench.bytes_per_token_head(WORKLOADS["fwd_bf16_d256"]) == 2 * (512 + 256) + 2 * 256 + 8
    assert bench.bytes_per_token_head(WORKLOADS["fwd_bf16_7b"]) == 4104
    w = WORKLOADS["fwd_bf16_long"]
    assert bench.bytes_per_token_head(w) == 4104
    fw = bench.fwd_work(w, True)
    tok = w.B * w.NH * w.S
    # the walk's algorithmic bytes are that figure times the token-heads of one launch: 4.30 GB at
    # 131072 tokens x 8 heads; the segment states it reads are reported apart, not counted
    assert fw["phases"]["outputs"]["bytes"] == 4104 * tok
    assert abs(fw["phases"]["outputs"]["bytes"] / 1e9 - 4.303) < 1e-3
    nseg = bench.segments(w)
    assert fw["phases"]["outputs"]["state_traffic"] == w.B * w.NH * nseg * 4 * (256 * 512 + 256)
    # the whole pass adds the final state written once
    assert fw["bytes"] == 4104 * tok + w.B * w.NH * 4 * (256 * 512 + 256 + 1)


def test_roofline_object():
    peaks = {"hbm_gbs": 6452.8, "bf16_tflops": 1662.0, "source": "measured"}
    r = bench.roofline({"bytes": 4.303e9, "flops": 6.5e11}, 1.0e-3, peaks, True)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 4303.0) < 1e-6 and abs(r["frac"] - 4303.0 / 6452.8) < 1e-12
    r = bench.roofline({"bytes": 1e6, "flops": 1.662e12}, 2.0e-3, peaks, True)
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12


def test_forward_flops_per_token_and_head():
    w = WORKLOADS["fwd_bf16_d256"]
    fw = bench.fwd_work(w, True)
    dk, dv, L = w.DHQK, w.DHV, w.chunk
    assert fw["flops"] == w.B * w.NH * w.S * (4 * dk * dv + (L + 1) * (dk + dv) + 4 * dk)


def test_decode_step_bytes_are_the_state_twice_plus_the_token():
    sw = bench.step_work(256, 8, 256, 512, e=2, ogate=True)
    heads = 256 * 8
    state = heads * 4 * (256 * 512 + 256 + 1)
    assert sw["bytes"] == 2 * state + heads * (2 * (2 * 256 + 512 + 512) + 8 + 2 * 512)
    assert sw["bytes"] > 2 * 2 ** 30          # the 1 GiB state read and written


def test_slstm_work():
    sw = bench.slstm_work(16, 1024, 4, 256, 4)
    assert sw["flops"] == 8 * 256 * 256 * 4 * 16 * 1024
    assert sw["bytes"] == 5 * 4 * 256 * 16 * 1024 * 4


def test_segment_planner_fills_whole_waves():
    # the library's planner (a host query): the bench workload's 16 heads x 2 value tiles and 32
    # chunks take four segments of eight chunks, 128 CTAs on the 148 SMs in one wave
    assert bench.segments(WORKLOADS["fwd_bf16_d256"]) == 4
    from xlstm_mlstm_cell_b200 import binding
    import torch
    for B, NH, S, DK, DV, L in [(1, 8, 8192, 256, 512, 64), (1, 8, 131072, 256, 512, 128), (1, 1, 512, 64, 128, 64),
                                (8, 8, 4096, 128, 512, 64), (2, 3, 333, 256, 256, 64)]:
        ns = binding.fwd_segments(B, NH, S, DK, DV, L, torch.bfloat16)
        NC = -(-S // L)
        R = -(-NC // ns)
        assert 1 <= ns <= min(NC, 256) and -(-NC // R) == ns
    # off the tensor-core path, or nothing to compute
    assert binding.fwd_segments(1, 8, 8192, 256, 512, 64, torch.float32) == 0
    assert binding.fwd_segments(1, 8, 8192, 96, 512, 64, torch.bfloat16) == 0
    assert binding.fwd_segments(0, 8, 8192, 256, 512, 64, torch.bfloat16) == 0
    assert binding.fwd_segments(1, 8, 0, 256, 512, 64, torch.bfloat16) == 0


def test_workload_overrides_for_captures():
    args = argparse.Namespace(workload="fwd_bf16_7b", seq=512, batch=64)
    w = bench.workload_for(args)
    assert (w.S, w.B) == (512, 64)
    assert dataclasses.replace(w, S=WORKLOADS["fwd_bf16_7b"].S, B=1) == WORKLOADS["fwd_bf16_7b"]
    args = argparse.Namespace(workload="fwd_bf16_d256", seq=0, batch=0)
    assert bench.workload_for(args) == WORKLOADS["fwd_bf16_d256"]
    # the headline workload is the largest forward configuration
    assert bench.DEFAULT_WORKLOAD == "fwd_bf16_long"


def test_whole_job_throughput():
    # N ranks x units per rank per step x steps over the slowest rank's time
    assert bench.job_throughput(4, 8196, 100, 50.0) == 4 * 8196 * 100 / 0.05
