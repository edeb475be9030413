"""The forget-gate gradient as a sum over token pairs, and the four groups the backward kernels sum.

Differentiating the read-out of the dual form ("The Dual Formulation: How mLSTM Enables Parallel
GPU Training", xLSTM Guide: Extended LSTM Architecture & Matrix Memory) through the decay weights
D_ts = exp(F_t - F_s + i~_s) (F the cumulative log forget gate): with R_ts = D_ts dL/dD_ts for
s <= t,

    dL/dlog f_j = sum over the pairs s < j <= t of R_ts,

since log f_j enters exactly the weights of those pairs.  These checks (numpy, fp64) pin:

* that pair sum, against the C adjoint oracle's d f~ = sigmoid(-f~) dL/dlog f;
* for j in chunk c, its split into four disjoint groups, the form the backward kernels compute:
  the pairs inside the chunk, the chunk's queries t >= j against earlier chunks, the chunk's
  keys s < j against later chunks, and E_c, the pairs that skip the chunk;
* E_c as the state inner product the kernels take, exp(g_c) (<G_{c+1}, C_c> + <dn_{c+1}, n_c>):
  the gradient of the state at the chunk's end against the decayed state at its start.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle


def _inputs(S, dk, dv, seed, ig, fg, qk_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, 1, S, dk, generator=g) * qk_scale
    k = torch.randn(1, 1, S, dk, generator=g) * qk_scale
    v = torch.randn(1, 1, S, dv, generator=g)
    i = torch.randn(1, 1, S, generator=g) * ig[1] + ig[0]
    f = torch.randn(1, 1, S, generator=g) * fg[1] + fg[0]
    o = torch.sigmoid(torch.randn(1, 1, S, dv, generator=g))
    dh = torch.randn(1, 1, S, dv, generator=g)
    return q, k, v, i, f, o, dh   # float32: the oracle and numpy see the same numbers


def _pairs(q, k, v, i, f, o, dh):
    """R [t][s] of one head from the unstabilized dual form (normalizer floored at 1), in fp64."""
    q, k, v, i, f, o, dh = (x[0, 0].double().numpy() for x in (q, k, v, i, f, o, dh))
    S, dk = q.shape
    scale = 1.0 / np.sqrt(dk)
    logf = -np.logaddexp(0.0, -f)                     # log sigmoid(f~)
    F = np.cumsum(logf)
    causal = np.tril(np.ones((S, S), dtype=bool))
    D = np.where(causal, np.exp(np.where(causal, F[:, None] - F[None, :] + i[None, :], 0.0)), 0.0)
    A = D * (q @ k.T) * scale
    num, den = A @ v, A.sum(axis=1)
    N = np.maximum(np.abs(den), 1.0)
    hh = num / N[:, None]
    g = o * dh / N[:, None]                           # dL/dnum
    dden = np.where(np.abs(den) > 1.0, -(g * hh).sum(axis=1) * np.sign(den), 0.0)
    R = A * (g @ v.T + dden[:, None])
    return R, dict(q=q, k=k, v=v, i=i, f=f, F=F, g=g, dden=dden, scale=scale)


def _straddling(R):
    S = R.shape[0]
    return np.array([R[j:, :j].sum() for j in range(S)])


CASES = [
    dict(S=23, dk=5, dv=4, seed=1, ig=(0.0, 1.0), fg=(2.0, 1.0)),
    dict(S=29, dk=4, dv=3, seed=2, ig=(0.0, 1.0), fg=(-4.0, 1.0)),              # strongly forgetting
    dict(S=26, dk=6, dv=5, seed=3, ig=(0.0, 1.0), fg=(3.0, 1.0), qk_scale=0.1),  # the floor binds
]


@pytest.mark.parametrize("case", CASES)
def test_pair_sum_is_the_forget_gate_gradient(case):
    inputs = _inputs(**case)
    R, x = _pairs(*inputs)
    ref = oracle.mlstm_adjoint(*inputs)[4][0, 0]       # d f~ from the C adjoint
    got = _straddling(R) / (1.0 + np.exp(x["f"]))      # sigmoid(-f~) dL/dlog f
    assert np.allclose(got, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max()), np.abs(got - ref).max()


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("L", [4, 5])
def test_four_groups_partition_the_straddling_pairs(case, L):
    R, x = _pairs(*_inputs(**case))
    S = R.shape[0]
    F_j = _straddling(R)
    q, k, v, i, F, g, dden, scale = (x[n] for n in ("q", "k", "v", "i", "F", "g", "dden", "scale"))
    for j in range(S):
        c = j // L
        t0, t1 = c * L, min((c + 1) * L, S)           # the chunk's tokens [t0, t1)
        e_c = R[t1:, :t0].sum()                        # pairs that skip the chunk
        q_inter = R[j:t1, :t0].sum()                   # its queries t >= j against earlier chunks
        k_inter = R[t1:, t0:j].sum()                   # its keys s < j against later chunks
        rect = R[j:t1, t0:j].sum()                     # pairs inside the chunk
        total = e_c + q_inter + k_inter + rect
        assert abs(total - F_j[j]) <= 1e-12 * max(1.0, np.abs(R).sum()), (j, total, F_j[j])
        # E_c from the states: the state after token t0 - 1 and the gradient of the state after
        # token t1 - 1, with the chunk's decay exp(F[t1 - 1] - F[t0 - 1]) between them
        if t0 > 0 and t1 < S:
            u = np.exp(F[t0 - 1] - F[:t0] + i[:t0])            # weights of the keys in C_c
            C_c, n_c = (u[:, None] * k[:t0]).T @ v[:t0], u @ k[:t0]
            w = np.exp(F[t1:] - F[t1 - 1]) * scale           # weights of the queries in G_{c+1}
            G_end, dn_end = (w[:, None] * q[t1:]).T @ g[t1:], (w * dden[t1:]) @ q[t1:]
            e_state = np.exp(F[t1 - 1] - F[t0 - 1]) * ((G_end * C_c).sum() + dn_end @ n_c)
            assert abs(e_state - e_c) <= 1e-12 * max(1.0, np.abs(R).sum()), (c, e_state, e_c)
        else:
            assert e_c == 0.0                          # no earlier or no later token
