"""mlstm_fwd_state (forward pass from a given state) against the fp64 oracle, through the C ABI.

The oracle runs the same token-by-token recurrence from the same initial state
(C0, n0, m0); the state itself comes from the oracle's own prefill of other
tokens, rounded to fp32, so that it has realistic magnitudes and stabilizer.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, assert_close, rel_l2
from xlstm_mlstm_cell_b200 import binding
from xlstm_mlstm_cell_b200.workloads import make_custom

pytestmark = pytest.mark.gpu


def oracle_state(B, NH, DK, DV, dt, seed):
    inp = make_custom(B, NH, 300, DK, DV, dt, seed=seed, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    _, C, n, m = oracle.run(*inp, want_h=False)
    return C.astype(np.float32), n.astype(np.float32), m.astype(np.float32)


@pytest.mark.parametrize("B,NH,S,DK,DV,chunk,dt", [
    (1, 2, 100, 16, 16, 16, "f32"), (2, 2, 333, 64, 48, 32, "f32"),
    (1, 2, 512, 256, 256, 64, "bf16"), (1, 2, 700, 256, 512, 128, "bf16"), (2, 1, 260, 128, 128, 64, "bf16"),
    (1, 2, 300, 64, 128, 64, "bf16")])
def test_fwd_from_state_matches_oracle(cuda_lib, B, NH, S, DK, DV, chunk, dt):
    C0, n0, m0 = oracle_state(B, NH, DK, DV, dt, seed=DK + S)
    inp = make_custom(B, NH, S, DK, DV, dt, seed=S + 5, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    g = [x.cuda() for x in inp]
    st = tuple(torch.from_numpy(x).cuda() for x in (C0, n0, m0))
    h, C, n, m = binding.fwd(*g, chunk=chunk, state=st)
    torch.cuda.synchronize()
    hr, Cr, nr, mr = oracle.run(*inp, C0, n0, m0)
    tol = TOL[dt]
    assert_close("h", h.cpu(), hr, tol)
    assert_close("C", C.cpu(), Cr, tol)
    assert_close("n", n.cpu(), nr, tol)
    assert_close("m", m.cpu(), mr, tol)


@pytest.mark.parametrize("dt,DK,DV,chunk", [("f32", 32, 32, 16), ("bf16", 256, 256, 64), ("bf16", 256, 512, 128)])
def test_split_prefill_equals_whole(cuda_lib, dt, DK, DV, chunk):
    """Prefill S1 tokens, then resume for S2 from the returned state == one pass over S1 + S2."""
    S1, S2 = 3 * chunk + 7, 2 * chunk + 11
    inp = [x.cuda() for x in make_custom(1, 2, S1 + S2, DK, DV, dt, seed=77, ig=(-1.0, 2.0), fg=(4.0, 1.0))]
    part = lambda x, a, b: x[:, :, a:b].contiguous()
    hw, Cw, nw, mw = binding.fwd(*inp, chunk=chunk)
    h1, C1, n1, m1 = binding.fwd(*[part(x, 0, S1) for x in inp], chunk=chunk)
    h2, C2, n2, m2 = binding.fwd(*[part(x, S1, S1 + S2) for x in inp], chunk=chunk, state=(C1, n1, m1))
    torch.cuda.synchronize()
    tol = TOL[dt]
    assert rel_l2(torch.cat([h1, h2], dim=2).cpu(), hw.cpu()) <= tol
    assert rel_l2(C2.cpu(), Cw.cpu()) <= tol and rel_l2(n2.cpu(), nw.cpu()) <= tol
    assert rel_l2(m2.cpu(), mw.cpu()) <= tol


@pytest.mark.parametrize("dt,DK,DV,chunk", [("f32", 32, 32, 16), ("bf16", 256, 256, 64)])
def test_state_updated_in_place(cuda_lib, dt, DK, DV, chunk):
    C0, n0, m0 = oracle_state(1, 2, DK, DV, dt, seed=3)
    inp = make_custom(1, 2, 257, DK, DV, dt, seed=9)
    Cg, ng, mg = (torch.from_numpy(x).cuda() for x in (C0, n0, m0))
    h, C, n, m = binding.fwd(*[x.cuda() for x in inp], chunk=chunk, state=(Cg, ng, mg), C_final=Cg, n_final=ng,
                             m_final=mg)
    torch.cuda.synchronize()
    hr, Cr, nr, mr = oracle.run(*inp, C0, n0, m0)
    tol = TOL[dt]
    assert_close("h", h.cpu(), hr, tol)
    assert_close("C in place", Cg.cpu(), Cr, tol)
    assert_close("n in place", ng.cpu(), nr, tol)
    assert_close("m in place", mg.cpu(), mr, tol)


def test_empty_sequence_returns_initial_state(cuda_lib):
    C0, n0, m0 = oracle_state(1, 2, 64, 64, "bf16", seed=4)
    inp = [x.cuda() for x in make_custom(1, 2, 0, 64, 64, "bf16", seed=1)]
    st = tuple(torch.from_numpy(x).cuda() for x in (C0, n0, m0))
    h, C, n, m = binding.fwd(*inp, chunk=64, state=st)
    torch.cuda.synchronize()
    assert torch.equal(C.cpu(), st[0].cpu()) and torch.equal(n.cpu(), st[1].cpu()) and torch.equal(m.cpu(), st[2].cpu())
