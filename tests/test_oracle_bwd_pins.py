"""Pins of the gradient oracle (oracle/mlstm_bwd.py).

* its forward recurrence equals the C oracle's h (which the other pins tie to the pages);
* central finite differences of that forward pass, for every input, with the denominator floor
  inactive and binding;
* dL/do = dh * h / o, since h is linear in the output gate;
* dL/dv from the causal decay matrix of the guide's dual form: h_t = o_t * sum_s W_ts v_s with
  W_ts = F_ts e^{i~_s} (qh_t . k_s) / max(|sum_s' F_ts' e^{i~_s'} (qh_t . k_s')|, 1) and F_ts the
  product of the forget gates after s up to t, so dL/dv_s = sum_t W_ts (dh_t * o_t).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import mlstm_bwd

NAMES = ("q", "k", "v", "igate", "fgate", "ogate")


def _inputs(B, NH, S, dk, dv, seed, scale=1.0, ogate=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, NH, S, dk, generator=g, dtype=torch.float64) * scale
    k = torch.randn(B, NH, S, dk, generator=g, dtype=torch.float64) * scale
    v = torch.randn(B, NH, S, dv, generator=g, dtype=torch.float64)
    i = torch.randn(B, NH, S, generator=g, dtype=torch.float64)
    f = torch.randn(B, NH, S, generator=g, dtype=torch.float64) + 2.0
    o = torch.sigmoid(torch.randn(B, NH, S, dv, generator=g, dtype=torch.float64)) if ogate else None
    dh = torch.randn(B, NH, S, dv, generator=g, dtype=torch.float64)
    # float32-representable values, so that the C oracle (float32 inputs) sees the same numbers
    rnd = lambda x: None if x is None else x.float().double()
    return tuple(rnd(x) for x in (q, k, v, i, f, o)), dh


def test_forward_matches_the_c_oracle():
    (q, k, v, i, f, o), _ = _inputs(2, 2, 23, 5, 4, seed=1)
    h64 = mlstm_bwd.mlstm_fwd64(q, k, v, i, f, o)
    hc, _, _, _ = oracle.run(q, k, v, i, f, o, nthreads=1)
    assert np.abs(h64 - hc).max() <= 1e-12 * np.abs(hc).max()


def _loss(xs, dh):
    with torch.no_grad():
        return float((mlstm_bwd.forward(*xs) * dh).sum())


@pytest.mark.parametrize("scale,floor_binds", [(1.5, False), (0.02, True)])
def test_finite_differences(scale, floor_binds):
    (q, k, v, i, f, o), dh = _inputs(1, 1, 6, 3, 2, seed=7, scale=scale)
    xs = [q, k, v, i, f, o]
    # which branch of the denominator's max the case exercises
    with torch.no_grad():
        lf = torch.nn.functional.logsigmoid(f)
        m = torch.zeros(1, 1, dtype=torch.float64)
        n = torch.zeros(1, 1, 3, dtype=torch.float64)
        binds = []
        for t in range(6):
            mn = torch.maximum(lf[..., t] + m, i[..., t])
            n = torch.exp(lf[..., t] + m - mn)[..., None] * n + torch.exp(i[..., t] - mn)[..., None] * k[..., t, :]
            binds.append(bool((torch.abs((n * q[..., t, :]).sum(-1) / math.sqrt(3)) < torch.exp(-mn)).all()))
            m = mn
    if floor_binds:
        assert all(binds)
    else:
        assert binds.count(False) >= 4          # mostly |n . qh| above the floor
    grads = mlstm_bwd.mlstm_bwd(q, k, v, i, f, o, dh)
    eps = 1e-6
    for idx, (name, x) in enumerate(zip(NAMES, xs)):
        fd = np.zeros(tuple(x.shape))
        flat = x.reshape(-1)
        for j in range(flat.numel()):
            xp = [y.clone() for y in xs]
            xm = [y.clone() for y in xs]
            xp[idx].reshape(-1)[j] += eps
            xm[idx].reshape(-1)[j] -= eps
            fd.reshape(-1)[j] = (_loss(xp, dh) - _loss(xm, dh)) / (2 * eps)
        g = grads[idx]
        err = np.abs(g - fd).max()
        assert err <= 1e-6 * max(1.0, np.abs(fd).max()), (name, err)


def test_output_gate_gradient_is_h_over_o():
    (q, k, v, i, f, o), dh = _inputs(2, 2, 9, 4, 3, seed=3)
    grads = mlstm_bwd.mlstm_bwd(q, k, v, i, f, o, dh)
    h = mlstm_bwd.mlstm_fwd64(q, k, v, i, f, o)
    assert np.abs(grads[5] - dh.numpy() * h / o.numpy()).max() <= 1e-12 * np.abs(grads[5]).max()


@pytest.mark.parametrize("scale", [1.0, 0.05])
def test_value_gradient_from_the_dual_form(scale):
    (q, k, v, i, f, o), dh = _inputs(1, 2, 11, 4, 3, seed=5, scale=scale)
    grads = mlstm_bwd.mlstm_bwd(q, k, v, i, f, o, dh)
    qn, kn, inn, fn, on, dhn = (x.numpy() for x in (q, k, i, f, o, dh))
    S, dk = qn.shape[2], qn.shape[3]
    dv_ref = np.zeros(v.shape)
    logsig = np.minimum(fn, 0.0) - np.log1p(np.exp(-np.abs(fn)))
    for hd in range(qn.shape[1]):
        cum = np.concatenate([[0.0], np.cumsum(logsig[0, hd])])          # cum[t + 1] = sum_{r <= t}
        W = np.zeros((S, S))
        for t in range(S):
            for s in range(t + 1):
                F = math.exp(cum[t + 1] - cum[s + 1])                     # forget gates s+1 .. t
                W[t, s] = F * math.exp(inn[0, hd, s]) * np.dot(qn[0, hd, t], kn[0, hd, s]) / math.sqrt(dk)
            W[t] /= max(abs(W[t].sum()), 1.0)
        dv_ref[0, hd] = W.T @ (dhn[0, hd] * on[0, hd])
    assert np.abs(grads[2] - dv_ref).max() <= 1e-11 * np.abs(dv_ref).max()


# ---------------------------------------------------------------- planted mistakes
# Mutated copies of the gradient oracle must fail at least one of the checks below: a slip in the
# forward shows against the C oracle, a cut gradient path against finite differences.  (Cutting
# the gradient through the stabilizer m is not a slip: h does not depend on m, so the gradient
# with m held fixed is the same.)

MUTATIONS = {
    "denominator_detached": ("den = torch.maximum(torch.abs((n * qh[..., t, :]).sum(-1)), torch.exp(-m_new))",
                             "den = torch.maximum(torch.abs((n * qh[..., t, :]).sum(-1)), torch.exp(-m_new)).detach()"),
    "no_q_scale": ("qh = q / math.sqrt(dk)", "qh = q"),
    "raw_forget_gate": ("lf = torch.nn.functional.logsigmoid(fgate)", "lf = fgate"),
    "normalizer_detached": ("n = fw[..., None] * n + iw[..., None] * k[..., t, :]",
                            "n = (fw[..., None] * n + iw[..., None] * k[..., t, :]).detach()"),
}


def _worst_check(mod):
    """Largest relative deviation of the forward check and of finite differences (both branches)."""
    (q, k, v, i, f, o), _ = _inputs(1, 2, 9, 3, 2, seed=11)
    hc, _, _, _ = oracle.run(q, k, v, i, f, o, nthreads=1)
    worst = np.abs(mod.mlstm_fwd64(q, k, v, i, f, o) - hc).max() / np.abs(hc).max()
    for scale in (1.5, 0.02):
        (q, k, v, i, f, o), dh = _inputs(1, 1, 5, 3, 2, seed=7, scale=scale)
        xs = [q, k, v, i, f, o]
        grads = mod.mlstm_bwd(q, k, v, i, f, o, dh)

        def loss(ys):
            with torch.no_grad():
                return float((mod.forward(*ys) * dh).sum())
        eps = 1e-6
        for idx, x in enumerate(xs):
            for j in range(x.numel()):
                xp = [y.clone() for y in xs]
                xm = [y.clone() for y in xs]
                xp[idx].reshape(-1)[j] += eps
                xm[idx].reshape(-1)[j] -= eps
                fd = (loss(xp) - loss(xm)) / (2 * eps)
                g = grads[idx].reshape(-1)[j]
                worst = max(worst, abs(g - fd) / max(1.0, abs(fd)))
    return worst


def test_checks_pass_for_the_oracle():
    assert _worst_check(mlstm_bwd) <= 1e-6


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation):
    src = open(mlstm_bwd.__file__).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) == 1, "mutation anchor not found: %s" % old
    import types
    mod = types.ModuleType("mlstm_bwd_mutant")
    exec(compile(src.replace(old, new), "mlstm_bwd_mutant.py", "exec"), mod.__dict__)
    assert _worst_check(mod) > 1e-4, mutation
