"""GPU parity of the sLSTM recurrence (slstm_fwd through the C ABI) against the fp64 oracle.

Shapes cover every supported head size (one to eight CTAs per cluster), batch sizes that leave the
last batch group ragged, both forget gates, a non-zero start state, fp32 (rel-L2 1e-5) and bf16
(rel-L2 1e-2) inputs; plus carrying the state across calls, the state-only call, and the bench
workload at full size with sampled batch items.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle.slstm import slstm_run
from tests.parity import TOL, assert_close
from xlstm_mlstm_cell_b200 import binding
from xlstm_mlstm_cell_b200.workloads import SLSTM_WORKLOADS, make_slstm_inputs

pytestmark = pytest.mark.gpu


# Forget-gate pre-activations ~ N(F_LOC[forget], 1).  With the exponential forget gate a positive
# mean would let the stabilizer m grow by about that much per step, and the fp32 rounding of a large
# m (not of the kernel) would then enter the input weights; the means keep m bounded, as a decaying
# memory does.
F_LOC = {"exp": -1.0, "sigmoid": 3.0}


def make_inputs(B, S, NH, DH, dt, seed, forget):
    """wx ~ N(0, 1) for i, z, o and N(F_LOC, 1) for f; R ~ N(0, 1 / DH) (R h of order one)."""
    return make_slstm_inputs(B, S, NH, DH, dt, seed, F_LOC[forget])


def make_state(B, NH, DH, seed):
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(B, NH, DH, generator=g)
    n = torch.rand(B, NH, DH, generator=g) + 0.5
    m = torch.randn(B, NH, DH, generator=g) * 0.5
    h = torch.tanh(torch.randn(B, NH, DH, generator=g))
    return c, n, m, h


def run_gpu(wx, R, forget, state=None, want_h=True):
    st = None if state is None else tuple(x.clone().cuda() for x in state)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    h, (c, n, m, hl) = binding.slstm_fwd(wx.cuda(), R.cuda(), forget=forget, state=st, want_h=want_h,
                                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "a bounded wait of the sLSTM kernel gave up"
    return (None if h is None else h.cpu()), (c.cpu(), n.cpu(), m.cpu(), hl.cpu())


@pytest.mark.parametrize("B,S,NH,DH,dt,forget", [
    (1, 1, 1, 32, "f32", "exp"),
    (3, 37, 2, 32, "f32", "sigmoid"),
    (5, 29, 1, 64, "f32", "exp"),
    (2, 33, 3, 128, "f32", "sigmoid"),
    (3, 21, 2, 192, "f32", "exp"),
    (2, 40, 2, 256, "f32", "sigmoid"),
    (9, 25, 2, 256, "bf16", "exp"),
    (4, 30, 3, 128, "bf16", "sigmoid"),
    (7, 18, 1, 64, "bf16", "exp"),
])
def test_slstm_matches_oracle(cuda_lib, B, S, NH, DH, dt, forget):
    wx, R = make_inputs(B, S, NH, DH, dt, seed=B * 100 + DH + S, forget=forget)
    state = make_state(B, NH, DH, seed=S)
    h, (c, n, m, hl) = run_gpu(wx, R, forget, state)
    hr, (cr, nr, mr, hlr) = slstm_run(wx, R, forget=forget, state=state)
    tol = TOL[dt]
    assert_close("h", h, hr, tol)
    assert_close("c", c, cr, tol)
    assert_close("n", n, nr, tol)
    assert_close("m", m, mr, tol)
    assert_close("h_last", hl, hlr, tol)


@pytest.mark.parametrize("B,NH,DH", [(1, 1, 256), (13, 3, 64), (37, 2, 128)])
def test_slstm_zero_start_and_batch_groups(cuda_lib, B, NH, DH):
    """A fresh sequence (all-zero state) for batch sizes that fill 1, 2, 4 or 8 items per cluster."""
    S = 17
    wx, R = make_inputs(B, S, NH, DH, "f32", seed=B + NH + DH, forget="exp")
    assert binding.slstm_batch_per_cluster(B, NH, DH, torch.float32) in (1, 2, 4, 8)
    h, (c, n, m, hl) = run_gpu(wx, R, "exp")
    hr, (cr, nr, mr, _) = slstm_run(wx, R, forget="exp")
    assert_close("h", h, hr, TOL["f32"])
    assert_close("c", c, cr, TOL["f32"])
    assert_close("n", n, nr, TOL["f32"])


def test_slstm_state_carries_across_calls(cuda_lib):
    B, S1, S2, NH, DH = 4, 19, 23, 2, 128
    wx, R = make_inputs(B, S1 + S2, NH, DH, "f32", seed=77, forget="sigmoid")
    h_all, st_all = run_gpu(wx, R, "sigmoid")
    h1, st1 = run_gpu(wx[:, :S1].contiguous(), R, "sigmoid")
    h2, st2 = run_gpu(wx[:, S1:].contiguous(), R, "sigmoid", state=st1)
    torch.testing.assert_close(torch.cat([h1, h2], dim=1), h_all, rtol=1e-6, atol=1e-6)
    for a, b in zip(st2, st_all):
        torch.testing.assert_close(a, b, rtol=1e-6, atol=1e-6)


def test_slstm_state_only_call(cuda_lib):
    B, S, NH, DH = 3, 31, 2, 64
    wx, R = make_inputs(B, S, NH, DH, "bf16", seed=5, forget="exp")
    _, st_a = run_gpu(wx, R, "exp")
    h, st_b = run_gpu(wx, R, "exp", want_h=False)
    assert h is None
    for a, b in zip(st_a, st_b):
        assert torch.equal(a, b)


def test_slstm_empty_sequence_is_a_no_op(cuda_lib):
    wx, R = make_inputs(2, 0, 1, 32, "f32", seed=1, forget="exp")
    state = make_state(2, 1, 32, seed=2)
    h, st = run_gpu(wx, R, "exp", state)
    assert h.shape == (2, 0, 1, 32)
    for a, b in zip(st, state):
        assert torch.equal(a, b)


def test_slstm_bench_workload_sampled(cuda_lib):
    """B16 S1024 NH4 DH256 fp32 (the benchmark's sLSTM workload) in one call; the oracle checks
    batch items 0 and 11 in full (batch items are independent)."""
    w = SLSTM_WORKLOADS["slstm_f32"]
    wx, R = make_slstm_inputs(w.B, w.S, w.NH, w.DH, w.dtype, w.seed, w.f_loc)
    h, (c, n, m, hl) = run_gpu(wx, R, w.forget)
    for b in (0, 11):
        hr, (cr, nr, mr, _) = slstm_run(wx[b:b + 1], R, forget=w.forget)
        assert_close("h[b=%d]" % b, h[b:b + 1], hr, TOL["f32"])
        assert_close("c[b=%d]" % b, c[b:b + 1], cr, TOL["f32"])
        assert_close("m[b=%d]" % b, m[b:b + 1], mr, TOL["f32"])
    assert np.isfinite(h.numpy()).all()
