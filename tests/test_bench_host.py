"""Host-side arithmetic of the benchmark (no GPU): the algorithmic work that the roofline fractions
divide by, and the workload overrides used by profiler captures."""
from __future__ import annotations

import argparse
import dataclasses

import bench
from xlstm_mlstm_cell_b200.workloads import WORKLOADS


def _walk_bytes_per_token_head(w):
    fw = bench.fwd_work(w, True)
    heads = w.B * w.NH
    nseg = bench.segments(w)
    state = heads * nseg * 4 * (w.DHQK * w.DHV + w.DHQK)
    return (fw["phases"]["outputs"]["bytes"] - state) / (heads * w.S)


def test_walk_bytes_per_token_and_head():
    # q, k, v (and o) read, h written, 12 bytes of gate values: 2 (2 dk + dv) + 2 dv [o] + 2 dv + 12
    assert _walk_bytes_per_token_head(WORKLOADS["fwd_bf16_d256"]) == 2 * (512 + 256) + 2 * 256 + 12
    assert _walk_bytes_per_token_head(WORKLOADS["fwd_bf16_7b"]) == 4108


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


def test_whole_job_throughput():
    # N ranks x units per rank per step x steps over the slowest rank's time
    assert bench.job_throughput(4, 8196, 100, 50.0) == 4 * 8196 * 100 / 0.05
