"""GPU parity of mlstm_step (one decode token, state in place) against the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, assert_close
from xlstm_mlstm_cell_b200 import binding
from xlstm_mlstm_cell_b200.workloads import WORKLOADS, draw, make_custom, make_step_inputs

pytestmark = pytest.mark.gpu


def oracle_prefill(B, NH, S, DHQK, DHV, dt, seed, **kw):
    inputs = make_custom(B, NH, S, DHQK, DHV, dt, seed=seed, **kw)
    _, C, n, m = oracle.run(*inputs, want_h=False)
    return C, n, m


def gpu_state(C, n, m):
    return (torch.from_numpy(C).float().cuda(), torch.from_numpy(n).float().cuda(),
            torch.from_numpy(m).float().cuda())


@pytest.mark.parametrize("B,NH,DHQK,DHV,dt", [
    (2, 3, 16, 16, "f32"), (1, 2, 64, 100, "f32"), (3, 2, 256, 512, "bf16"), (2, 2, 128, 1024, "bf16"),
    (1, 1, 8, 4, "f32"), (4, 1, 512, 256, "bf16"), (10, 8, 64, 64, "f32")])
def test_step_chain(cuda_lib, B, NH, DHQK, DHV, dt):
    """Ten steps in a row from an oracle-made state; every h and the final state match."""
    C, n, m = oracle_prefill(B, NH, 40, DHQK, DHV, dt, seed=DHQK + DHV, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    Cg, ng, mg = gpu_state(C, n, m)
    Cr, nr, mr = C.astype(np.float32).astype(np.float64), n.astype(np.float32).astype(np.float64), \
        m.astype(np.float32).astype(np.float64)
    tol = TOL[dt]
    gen = torch.Generator().manual_seed(77)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    for s in range(10):
        q, k, v, i, f, o = draw((B, NH, DHQK), (B, NH, DHV), (B, NH), tdt, 1.0, (-1.0, 2.0), (4.0, 1.0), True, gen)
        h = binding.step(Cg, ng, mg, q.cuda(), k.cuda(), v.cuda(), i.cuda(), f.cuda(), o.cuda())
        hr, Cr, nr, mr = oracle.mlstm_step(Cr, nr, mr, q, k, v, i, f, o)
        assert_close("h step %d" % s, h.cpu(), hr, tol)
    torch.cuda.synchronize()
    assert_close("C", Cg.cpu(), Cr, tol)
    assert_close("n", ng.cpu(), nr, tol)
    assert_close("m", mg.cpu(), mr, tol)


def test_step_without_output_gate(cuda_lib):
    C, n, m = oracle_prefill(2, 2, 16, 64, 64, "bf16", seed=3)
    Cg, ng, mg = gpu_state(C, n, m)
    q, k, v, i, f, _ = make_custom(2, 2, 1, 64, 64, "bf16", seed=4)
    sq = lambda x: x[:, :, 0].contiguous()
    h = binding.step(Cg, ng, mg, sq(q).cuda(), sq(k).cuda(), sq(v).cuda(), sq(i).cuda(), sq(f).cuda(), None)
    hr, Cr, nr, mr = oracle.mlstm_step(C.astype(np.float32), n.astype(np.float32), m.astype(np.float32),
                                       sq(q), sq(k), sq(v), sq(i), sq(f), None)
    assert_close("h", h.cpu(), hr, TOL["bf16"])
    assert_close("C", Cg.cpu(), Cr, TOL["bf16"])


def prefill_state_full(w):
    """The decode workload's state: the oracle's fp64 prefill of 512 tokens, rounded to fp32.

    Drawn per batch element (seed derived from the workload seed and b) to bound host memory.
    """
    Cs = np.empty((w.B, w.NH, w.DHQK, w.DHV), dtype=np.float32)
    ns = np.empty((w.B, w.NH, w.DHQK), dtype=np.float32)
    ms = np.empty((w.B, w.NH), dtype=np.float32)
    step = 32
    for b0 in range(0, w.B, step):
        gen = torch.Generator().manual_seed(w.seed * 1000 + b0)
        inputs = draw((step, w.NH, w.S, w.DHQK), (step, w.NH, w.S, w.DHV), (step, w.NH, w.S), w.torch_dtype,
                      w.qkv_scale, w.ig, w.fg, w.ogate, gen)
        _, C, n, m = oracle.run(*inputs, want_h=False)
        Cs[b0:b0 + step], ns[b0:b0 + step], ms[b0:b0 + step] = C, n, m
    return Cs, ns, ms


def test_step_full_workload(cuda_lib):
    """B256 NH8 d256/512 state from the oracle's 512-token prefill; 1000 steps on all 2048 heads.

    h of every head is compared at every step, and the whole state after step 1000.
    """
    w = WORKLOADS["step_bf16"]
    Cs, ns, ms = prefill_state_full(w)
    Cg, ng, mg = (torch.from_numpy(x).cuda() for x in (Cs, ns, ms))
    Cr, nr, mr = (np.ascontiguousarray(x, dtype=np.float64) for x in (Cs, ns, ms))
    del Cs
    tol = TOL[w.dtype]
    worst = 0.0
    for s in range(w.steps):
        q, k, v, i, f, o = make_step_inputs(w, s)
        h = binding.step(Cg, ng, mg, q.cuda(), k.cuda(), v.cuda(), i.cuda(), f.cuda(), o.cuda())
        hr, _, _, _ = oracle.mlstm_step(Cr, nr, mr, q, k, v, i, f, o, inplace=True)
        worst = max(worst, assert_close("h step %d" % s, h.cpu(), hr, tol))
    torch.cuda.synchronize()
    assert_close("C after %d steps" % w.steps, Cg.cpu(), Cr, tol)
    assert_close("n after %d steps" % w.steps, ng.cpu(), nr, tol)
    assert_close("m after %d steps" % w.steps, mg.cpu(), mr, tol)
