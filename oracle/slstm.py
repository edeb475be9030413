"""fp64 CPU oracle of the sLSTM cell's recurrence (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this module; the CUDA library and its binding never do.

What it follows: "xLSTM Guide: Extended LSTM Architecture & Matrix Memory",
section "The Twin Cells: sLSTM and mLSTM Mathematical Formulations", part 1
"sLSTM: Scalar Memory with Recurrent Cross-Head Mixing" (the step-by-step
recurrent equations), read together with the hu-po summary "Introduction to
xLSTM architecture", section "xLSTM Architecture Design" (the residual block
with post-up projection), which says that the sLSTM's cell input and gates pass
through a block-diagonal linear layer of four diagonal blocks, its "heads", so
that connectivity stays inside each head.  The guide's title speaks of mixing
across heads; the hu-po statement is taken (R is block-diagonal over heads);
with one head the two agree.

Per batch item, head and cell j, at step t (1-based), from the state
(c, n, m, h) of step t-1:

* pre-activations: x~_t[g, j] = wx_t[g, j] + sum_k R[g, j, k] h_{t-1}[k] for the
  gates g = i, f, z, o; wx_t is W x_t + b (the input projection, computed
  outside the recurrence) and R is the head's recurrent matrix, one DH x DH
  block per gate (block-diagonal over heads);
* log forget gate: lf = f~ for the exponential forget gate (the equations of
  the page: m_t = max(m_{t-1} + f~_t, i~_t)), or lf = log sigmoid(f~) for the
  sigmoid forget gate that the paper also allows;
* stabilizer m_t = max(lf + m_{t-1}, i~_t);
* c_t = exp(lf + m_{t-1} - m_t) c_{t-1} + exp(i~_t - m_t) tanh(z~_t);
* n_t = exp(lf + m_{t-1} - m_t) n_{t-1} + exp(i~_t - m_t);
* h_t = sigmoid(o~_t) c_t / n_t.

Readings where the pages leave a step open: the state starts from the values
passed in (all zero for a fresh sequence, m_0 = 0 as for the mLSTM cell); R[g]
multiplies h_{t-1} as R[g] @ h_{t-1} (row j of R[g] feeds cell j).

Layouts: wx [B, S, 4, NH, DH] (gate order i, f, z, o); R [NH, 4, DH, DH];
state c, n, m, h [B, NH, DH]; outputs h_seq [B, S, NH, DH].  Inputs are widened
to float64 exactly (fp32 or bf16 data); the arithmetic is float64 throughout.

Parity pins (tests/test_oracle_pins_slstm.py): hand-derived values for two tiny
cases (tests/golden/slstm_hand_*.json), the closed form of equal gates (a
running mean of tanh(z~)), the stabilizer's cancellation in c / n, the feedback
decomposition of R, and the independence of heads.
"""
from __future__ import annotations

import numpy as np

GATES = ("i", "f", "z", "o")


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):                     # a torch tensor: widen on the CPU
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def log_sigmoid(x):
    """log(1 / (1 + e^-x)) without overflow: min(x, 0) - log1p(e^-|x|)."""
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    return np.exp(log_sigmoid(x))


def slstm_run(wx, R, forget="exp", state=None):
    """Runs the recurrence over all S steps.

    wx: [B, S, 4, NH, DH] pre-activations W x_t + b; R: [NH, 4, DH, DH];
    forget: "exp" (log forget gate = f~) or "sigmoid" (log forget gate =
    log sigmoid(f~)); state: (c, n, m, h), each [B, NH, DH], or None for zeros.
    Returns h_seq [B, S, NH, DH] and the state after the last step, float64.
    """
    if forget not in ("exp", "sigmoid"):
        raise ValueError("forget must be 'exp' or 'sigmoid'")
    wx, R = _f64(wx), _f64(R)
    B, S, four, NH, DH = wx.shape
    assert four == 4 and R.shape == (NH, 4, DH, DH)
    if state is None:
        c, n, m, h = (np.zeros((B, NH, DH)) for _ in range(4))
    else:
        c, n, m, h = (_f64(s).copy() for s in state)
    h_seq = np.zeros((B, S, NH, DH))
    for t in range(S):
        # recurrent term, one matrix-vector product per (batch item, head, gate)
        rec = np.einsum("egjk,bek->bgej", R, h)              # [B, 4, NH, DH]
        pre = wx[:, t] + rec
        ig, fg, zg, og = pre[:, 0], pre[:, 1], pre[:, 2], pre[:, 3]
        lf = fg if forget == "exp" else log_sigmoid(fg)
        m_new = np.maximum(lf + m, ig)
        fw = np.exp(lf + m - m_new)
        iw = np.exp(ig - m_new)
        c = fw * c + iw * np.tanh(zg)
        n = fw * n + iw
        h = sigmoid(og) * c / n
        m = m_new
        h_seq[:, t] = h
    return h_seq, (c, n, m, h)
