"""GPU parity of the sequence-parallel pieces (mlstm_fwd_final_state, mlstm_log_decay_sum,
mlstm_state_prefix) through the C ABI, with R ranks emulated one after the other on one
GPU (the all-gather replaced by stacking): the slices' h and the last slice's state must
match the oracle's single pass over the whole sequence.
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


def _logsigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


@pytest.mark.parametrize("R,B,NH,S,DK,DV,chunk,dt", [
    (2, 1, 2, 256, 16, 16, 16, "f32"),
    (3, 1, 2, 3 * 200, 256, 256, 64, "bf16"),
    (4, 1, 2, 4 * 256, 256, 512, 128, "bf16"),
    (2, 2, 1, 2 * 333, 128, 128, 64, "bf16"),
])
def test_sequence_parallel_equals_one_pass(cuda_lib, R, B, NH, S, DK, DV, chunk, dt):
    q, k, v, i, f, o = make_custom(B, NH, S, DK, DV, dt, seed=R * 7 + DK, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    L = S // R
    cut = lambda x, r: x[:, :, r * L:(r + 1) * L].contiguous().cuda()
    summaries = []
    for r in range(R):
        C_r, n_r, m_r = binding.fwd_final_state(cut(k, r), cut(v, r), cut(i, r), cut(f, r), chunk=chunk)
        summaries.append((C_r, n_r, m_r, binding.log_decay_sum(cut(f, r))))
    C_parts, n_parts, m_parts, g_parts = (torch.stack([s[j] for s in summaries]) for j in range(4))
    hs = []
    for r in range(R):
        start = binding.state_prefix(C_parts, n_parts, m_parts, g_parts, r)
        h, C, n, m = binding.fwd(cut(q, r), cut(k, r), cut(v, r), cut(i, r), cut(f, r), cut(o, r), chunk=chunk,
                                 state=start)
        hs.append(h)
    torch.cuda.synchronize()
    hr, Cr, nr, mr = oracle.mlstm_fwd(q, k, v, i, f, o)
    assert_close("h", torch.cat([x.cpu() for x in hs], dim=2), hr, TOL[dt])
    m64 = m.cpu().double().numpy()
    eC = np.exp(m64)[..., None, None] * C.cpu().double().numpy()
    en = np.exp(m64)[..., None] * n.cpu().double().numpy()
    assert rel_l2(eC, np.exp(mr)[..., None, None] * Cr) <= TOL[dt]
    assert rel_l2(en, np.exp(mr)[..., None] * nr) <= TOL[dt]


def test_final_state_pieces(cuda_lib):
    """mlstm_fwd_final_state gives mlstm_fwd's final state; the log decay sums match the
    oracle's logsigmoid; rank 0's start state is the zero state."""
    q, k, v, i, f, o = make_custom(2, 2, 777, 256, 256, "bf16", seed=5, ig=(-1.0, 2.0), fg=(4.0, 1.0))
    dev = [x.cuda() for x in (q, k, v, i, f, o)]
    _, C1, n1, m1 = binding.fwd(*dev, chunk=64)
    C2, n2, m2 = binding.fwd_final_state(dev[1], dev[2], dev[3], dev[4], chunk=64)
    g = binding.log_decay_sum(dev[4])
    torch.cuda.synchronize()
    assert torch.equal(C1, C2) and torch.equal(n1, n2) and torch.equal(m1, m2)
    gr = _logsigmoid(f.numpy()).sum(-1)
    assert np.abs(g.cpu().double().numpy() - gr).max() <= 1e-5 * np.abs(gr).max()
    parts = [x.unsqueeze(0) for x in (C1, n1, m1, g)]
    C0, n0, m0 = binding.state_prefix(*parts, 0)
    torch.cuda.synchronize()
    assert not C0.any() and not n0.any() and not m0.any()
