"""Pins of the sLSTM oracle (oracle/slstm.py) to facts that do not come from the oracle itself.

* hand-derived values for two tiny cases (tests/golden/slstm_hand_*.json): memory mixing through
  an asymmetric R (a transposed R fails), the stabilizer shifting between steps, an exponential
  forget gate above 1, and the sigmoid forget gate;
* closed form: with i~ = f~ = 0 (exponential forget) and R = 0 every weight is 1, so
  h_t = sigmoid(o~_t) * mean_{s<=t} tanh(z~_s);
* the stabilizer cancels in c / n: the unstabilized recurrence (plain exponentials, moderate gates)
  gives the same h;
* feedback decomposition: the run with R equals the run with R = 0 whose pre-activations have
  R[g] @ h_{t-1} added, h_{t-1} taken from the first run's output (pins the row / column roles of R);
* heads do not mix: changing one head's inputs or weights leaves the other heads' outputs unchanged;
* a state carried over: running S1 then S2 steps from the carried state equals one run of S1 + S2.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

from oracle.slstm import slstm_run

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng, loc=0.0, scale=1.0):
    # float32 values, as the library receives them
    return (rng.standard_normal(shape) * scale + loc).astype(np.float32)


@pytest.mark.parametrize("name", ["slstm_hand_mixing_three_steps.json", "slstm_hand_sigmoid_forget.json"])
def test_hand_derived(name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    wx = np.asarray(g["wx"], dtype=np.float32)[None]          # [1, S, 4, NH, DH]
    R = np.asarray(g["R"], dtype=np.float32)
    h_seq, (c, n, m, h) = slstm_run(wx, R, forget=g["forget"])
    tol = g["tol"]
    np.testing.assert_allclose(h_seq[0, :, 0], np.asarray(g["h_expected"]), rtol=tol, atol=tol)
    np.testing.assert_allclose(c[0, 0], g["c_expected"], rtol=tol, atol=tol)
    np.testing.assert_allclose(n[0, 0], g["n_expected"], rtol=tol, atol=tol)
    np.testing.assert_allclose(m[0, 0], g["m_expected"], rtol=tol, atol=tol)
    np.testing.assert_allclose(h[0, 0], np.asarray(g["h_expected"])[-1], rtol=tol, atol=tol)


def test_equal_gates_average_the_cell_inputs():
    rng = np.random.default_rng(1)
    B, S, NH, DH = 2, 9, 2, 3
    wx = np.zeros((B, S, 4, NH, DH), np.float32)
    wx[:, :, 2] = _rand((B, S, NH, DH), rng)
    wx[:, :, 3] = _rand((B, S, NH, DH), rng)
    h_seq, _ = slstm_run(wx, np.zeros((NH, 4, DH, DH), np.float32), forget="exp")
    z = wx[:, :, 2].astype(np.float64)
    o = wx[:, :, 3].astype(np.float64)
    mean_tanh = np.cumsum(np.tanh(z), axis=1) / np.arange(1, S + 1)[None, :, None, None]
    expect = mean_tanh / (1.0 + np.exp(-o))
    np.testing.assert_allclose(h_seq, expect, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("forget", ["exp", "sigmoid"])
def test_stabilizer_cancels(forget):
    """Without the stabilizer: c_t = F c + e^{i~} tanh(z~), n_t = F n + e^{i~}, F = e^{f~} or sigmoid(f~)."""
    rng = np.random.default_rng(2)
    B, S, NH, DH = 1, 12, 2, 4
    wx = _rand((B, S, 4, NH, DH), rng, scale=0.8)
    R = _rand((NH, 4, DH, DH), rng, scale=0.3)
    h_seq, _ = slstm_run(wx, R, forget=forget)
    w64, R64 = wx.astype(np.float64), R.astype(np.float64)
    c = np.zeros((B, NH, DH))
    n = np.zeros((B, NH, DH))
    h = np.zeros((B, NH, DH))
    for t in range(S):
        pre = w64[:, t].copy()
        for e in range(NH):
            for g in range(4):
                pre[:, g, e] += h[:, e] @ R64[e, g].T
        F = np.exp(pre[:, 1]) if forget == "exp" else 1.0 / (1.0 + np.exp(-pre[:, 1]))
        c = F * c + np.exp(pre[:, 0]) * np.tanh(pre[:, 2])
        n = F * n + np.exp(pre[:, 0])
        h = c / n / (1.0 + np.exp(-pre[:, 3]))
        np.testing.assert_allclose(h_seq[:, t], h, rtol=1e-11, atol=1e-13)


def test_feedback_decomposition():
    rng = np.random.default_rng(3)
    B, S, NH, DH = 2, 7, 2, 5
    wx = _rand((B, S, 4, NH, DH), rng)
    R = _rand((NH, 4, DH, DH), rng, scale=0.5)
    h_seq, _ = slstm_run(wx, R, forget="sigmoid")
    fed = wx.astype(np.float64)
    for t in range(1, S):
        for e in range(NH):
            for g in range(4):
                # row j of R[e, g] feeds cell j: (R @ h)[j] = sum_k R[j, k] h[k]
                fed[:, t, g, e] += np.stack([R[e, g].astype(np.float64) @ h_seq[b, t - 1, e] for b in range(B)])
    h2, _ = slstm_run(fed, np.zeros_like(R), forget="sigmoid")
    np.testing.assert_allclose(h2, h_seq, rtol=1e-12, atol=1e-14)
    # the transposed reading is a different function on this input
    h3, _ = slstm_run(wx, np.swapaxes(R, 2, 3), forget="sigmoid")
    assert np.abs(h3 - h_seq).max() > 1e-3


def test_heads_do_not_mix():
    rng = np.random.default_rng(4)
    B, S, NH, DH = 1, 6, 3, 4
    wx = _rand((B, S, 4, NH, DH), rng)
    R = _rand((NH, 4, DH, DH), rng, scale=0.5)
    h_a, _ = slstm_run(wx, R)
    wx2, R2 = wx.copy(), R.copy()
    wx2[:, :, :, 1] += 1.0
    R2[1] *= -1.0
    h_b, _ = slstm_run(wx2, R2)
    assert np.array_equal(h_a[:, :, [0, 2]], h_b[:, :, [0, 2]])
    assert np.abs(h_a[:, :, 1] - h_b[:, :, 1]).max() > 1e-3


def test_carried_state_continues_the_sequence():
    rng = np.random.default_rng(5)
    B, S1, S2, NH, DH = 2, 5, 4, 2, 3
    wx = _rand((B, S1 + S2, 4, NH, DH), rng)
    R = _rand((NH, 4, DH, DH), rng, scale=0.5)
    h_all, st_all = slstm_run(wx, R, forget="exp")
    h1, st1 = slstm_run(wx[:, :S1], R, forget="exp")
    h2, st2 = slstm_run(wx[:, S1:], R, forget="exp", state=st1)
    np.testing.assert_array_equal(np.concatenate([h1, h2], axis=1), h_all)
    for a, b in zip(st2, st_all):
        np.testing.assert_array_equal(a, b)


def test_rejects_unknown_forget_gate():
    with pytest.raises(ValueError):
        slstm_run(np.zeros((1, 1, 4, 1, 1), np.float32), np.zeros((1, 4, 1, 1), np.float32), forget="tanh")


def test_sigmoid_helpers_are_stable():
    from oracle.slstm import log_sigmoid
    x = np.array([-800.0, -30.0, 0.0, 30.0, 800.0])
    ls = log_sigmoid(x)
    assert np.all(np.isfinite(ls))
    assert ls[2] == -math.log(2.0)
    assert ls[0] == -800.0 and ls[4] == 0.0


# ---------------------------------------------------------------- planted mistakes
# Mutated copies of the oracle (one plausible slip each) must fail at least one pin.

MUTATIONS = {
    "transposed_R": ('rec = np.einsum("egjk,bek->bgej", R, h)', 'rec = np.einsum("egkj,bek->bgej", R, h)'),
    "heads_mix": ('rec = np.einsum("egjk,bek->bgej", R, h)', 'rec = np.einsum("egjk,bfk->bgej", R, h)'),
    "forget_ignores_stabilizer": ("fw = np.exp(lf + m - m_new)", "fw = np.exp(lf)"),
    "normalizer_drops_input": ("n = fw * n + iw", "n = fw * n + 1.0"),
    "no_tanh_on_z": ("c = fw * c + iw * np.tanh(zg)", "c = fw * c + iw * zg"),
    "raw_output_gate": ("h = sigmoid(og) * c / n", "h = og * c / n"),
    "sigmoid_forget_as_exp": ('lf = fg if forget == "exp" else log_sigmoid(fg)', "lf = fg"),
}


def pin_errors(run):
    """Largest deviation of each pin for an implementation `run` with slstm_run's signature."""
    errs = {}
    for name in ("slstm_hand_mixing_three_steps.json", "slstm_hand_sigmoid_forget.json"):
        g = json.load(open(os.path.join(GOLDEN, name)))
        wx = np.asarray(g["wx"], dtype=np.float32)[None]
        h_seq, (c, n, m, h) = run(wx, np.asarray(g["R"], dtype=np.float32), forget=g["forget"])
        errs[name] = max(np.abs(h_seq[0, :, 0] - np.asarray(g["h_expected"])).max(),
                         np.abs(c[0, 0] - g["c_expected"]).max(), np.abs(n[0, 0] - g["n_expected"]).max())
    rng = np.random.default_rng(2)
    B, S, NH, DH = 1, 12, 2, 4
    wx = _rand((B, S, 4, NH, DH), rng, scale=0.8)
    R = _rand((NH, 4, DH, DH), rng, scale=0.3)
    for forget in ("exp", "sigmoid"):
        h_seq, _ = run(wx, R, forget=forget)
        w64, R64 = wx.astype(np.float64), R.astype(np.float64)
        c = np.zeros((B, NH, DH))
        n = np.zeros((B, NH, DH))
        h = np.zeros((B, NH, DH))
        worst = 0.0
        for t in range(S):
            pre = w64[:, t].copy()
            for e in range(NH):
                for g in range(4):
                    pre[:, g, e] += h[:, e] @ R64[e, g].T
            F = np.exp(pre[:, 1]) if forget == "exp" else 1.0 / (1.0 + np.exp(-pre[:, 1]))
            c = F * c + np.exp(pre[:, 0]) * np.tanh(pre[:, 2])
            n = F * n + np.exp(pre[:, 0])
            h = c / n / (1.0 + np.exp(-pre[:, 3]))
            worst = max(worst, np.abs(h_seq[:, t] - h).max())
        errs["unstabilized_" + forget] = worst
    return errs


def test_pins_hold_for_the_oracle():
    errs = pin_errors(slstm_run)
    assert max(errs.values()) <= 1e-6, errs


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation):
    import oracle.slstm as mod
    src = open(mod.__file__).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) == 1, "mutation anchor not found: %s" % old
    ns = {"__name__": "slstm_mutant"}
    exec(compile(src.replace(old, new), "slstm_mutant.py", "exec"), ns)
    errs = pin_errors(ns["slstm_run"])
    assert max(errs.values()) > 1e-4, (mutation, errs)
