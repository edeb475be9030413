"""Failure detection on the GPU without a fault: a bounded device-side wait that runs out
is reported as MLSTM_ERR_TIMEOUT through the workspace's status word, and the context
stays usable for the next call.

mlstm_selftest_wait_timeout makes one CTA wait, through the kernels' own bounded wait,
on an mbarrier that nothing completes (a flag that nothing sets); the wait gives up
after its 2 s limit.
"""
from __future__ import annotations

import time

import pytest
import torch

import oracle
from tests.parity import TOL, assert_close
from xlstm_mlstm_cell_b200 import binding
from xlstm_mlstm_cell_b200.workloads import make_custom

pytestmark = pytest.mark.gpu

CODE = {name: code for code, name in binding.STATUS.items()}


def test_timed_out_wait_is_reported_and_the_context_stays_usable(cuda_lib):
    lib = binding.load()
    B, NH, S, DK, DV, chunk = 1, 2, 300, 128, 128, 64
    ws = binding.alloc_workspace(B, NH, S, DK, DV, chunk, torch.bfloat16, "cuda")
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t0 = time.time()
    assert lib.mlstm_selftest_wait_timeout(ws.data_ptr(), stream.cuda_stream) == CODE["MLSTM_OK"]
    assert binding.fwd_status(ws) == CODE["MLSTM_ERR_TIMEOUT"]
    elapsed = time.time() - t0
    assert 1.5 < elapsed < 30.0, elapsed          # the wait's limit is 2 s

    # the next call on the same workspace resets the status word and computes correctly
    inputs = make_custom(B, NH, S, DK, DV, "bf16", seed=9, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    q, k, v, i, f, o = (x.cuda() for x in inputs)
    h, C, n, m = binding.fwd(q, k, v, i, f, o, chunk=chunk, workspace=ws)
    assert binding.fwd_status(ws) == CODE["MLSTM_OK"]
    hr, Cr, nr, mr = oracle.mlstm_fwd(*inputs)
    assert_close("h", h.cpu(), hr, TOL["bf16"])
    assert_close("C", C.cpu(), Cr, TOL["bf16"])


def test_selftest_rejects_bad_workspace(cuda_lib):
    lib = binding.load()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.mlstm_selftest_wait_timeout(None, stream) == CODE["MLSTM_ERR_INVALID_ARG"]
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    assert lib.mlstm_selftest_wait_timeout(ws.data_ptr() + 16, stream) == \
        CODE["MLSTM_ERR_INVALID_ARG"]
