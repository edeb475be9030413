"""fp64 CPU oracle of the mLSTM forward pass's gradients (test infrastructure only).

Only the tests may import this module; the CUDA library and its binding never do.  No kernel of
the library computes these gradients yet: this is the reference a chunkwise backward pass will be
checked against.

Definition.  The forward pass is the stabilized recurrence of "xLSTM Guide: Extended LSTM
Architecture & Matrix Memory" ("The Stabilizer State", "Recurrent Formulation (Inference
Mode)"), read as the library reads it: log f = logsigmoid(f~), m_t = max(log f_t + m_{t-1}, i~_t),
f' = exp(log f_t + m_{t-1} - m_t), i' = exp(i~_t - m_t), C_t = f' C_{t-1} + i' k_t v_t^T,
n_t = f' n_{t-1} + i' k_t, h_t = o_t * (C_t^T qh_t) / max(|n_t . qh_t|, exp(-m_t)),
qh = q / sqrt(DHQK), from the zero state.  It is written here token by token with plain torch
float64 operations, and the gradients of a loss L = sum(dh * h) with respect to q, k, v, i~, f~
and o are torch.autograd's derivatives of exactly that computation (the library primitive that
differentiates it; no step is reordered or fused).  h does not depend on the stabilizer: in
unstabilized terms h = o * (Cbar^T qh) / max(|nbar . qh|, 1), so the gradient paths through m
cancel (holding m fixed gives the same gradient).  The derivative of the max in the denominator
is taken on the branch the forward pass picked.

Pins (tests/test_oracle_bwd_pins.py): the forward part against the C oracle; central finite
differences of that forward pass for every input; dL/do = dh * h / o (h is linear in o); dL/dv
from the causal decay matrix of the guide's dual form (h is linear in v for fixed gates, q and
k); planted mistakes that must fail them.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _t64(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).clone()
    return torch.tensor(np.asarray(x, dtype=np.float64))


def forward(q, k, v, igate, fgate, ogate=None):
    """The recurrence in float64 torch ops (differentiable): h [B, NH, S, DHV]."""
    B, NH, S, dk = q.shape
    dv = v.shape[-1]
    C = torch.zeros(B, NH, dk, dv, dtype=torch.float64)
    n = torch.zeros(B, NH, dk, dtype=torch.float64)
    m = torch.zeros(B, NH, dtype=torch.float64)
    qh = q / math.sqrt(dk)
    lf = torch.nn.functional.logsigmoid(fgate)
    hs = []
    for t in range(S):
        m_new = torch.maximum(lf[..., t] + m, igate[..., t])
        fw = torch.exp(lf[..., t] + m - m_new)
        iw = torch.exp(igate[..., t] - m_new)
        C = fw[..., None, None] * C + iw[..., None, None] * (k[..., t, :, None] * v[..., t, None, :])
        n = fw[..., None] * n + iw[..., None] * k[..., t, :]
        num = torch.einsum("bhkv,bhk->bhv", C, qh[..., t, :])
        den = torch.maximum(torch.abs((n * qh[..., t, :]).sum(-1)), torch.exp(-m_new))
        h = num / den[..., None]
        if ogate is not None:
            h = ogate[..., t, :] * h
        hs.append(h)
        m = m_new
    return torch.stack(hs, dim=2)


def mlstm_bwd(q, k, v, igate, fgate, ogate, dh):
    """Gradients of sum(dh * h) w.r.t. (q, k, v, igate, fgate, ogate), float64 numpy arrays
    (the ogate entry is None when ogate is None)."""
    xs = [_t64(x) for x in (q, k, v, igate, fgate, ogate)]
    for x in xs:
        if x is not None:
            x.requires_grad_(True)
    h = forward(*xs)
    loss = (h * _t64(dh)).sum()
    leaves = [x for x in xs if x is not None]
    grads = torch.autograd.grad(loss, leaves)
    out, it = [], iter(grads)
    for x in xs:
        out.append(None if x is None else next(it).numpy())
    return tuple(out)


def mlstm_fwd64(q, k, v, igate, fgate, ogate=None):
    """h of the forward pass (float64 numpy) from the same torch recurrence."""
    with torch.no_grad():
        return forward(*[_t64(x) for x in (q, k, v, igate, fgate, ogate)]).numpy()
