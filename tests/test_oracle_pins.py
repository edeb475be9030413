"""Pins the fp64 oracle to results fixed by the mathematics, not by itself.

Each check below evaluates the cell a second, independent way (numpy, fp64)
and compares it with the oracle:

* the closed (unrolled) form of the memory, C_t = sum_i (prod_{j>i} f_j) i_i k_i v_i^T,
  from the xLSTM tutorial's "Parallel Scan for mLSTM" formula (nareshka.ru
  "xLSTM: расширенная архитектура долгой краткосрочной памяти", section
  "Параллелизация"), with the normalizer summed the same way;
* an unstabilized evaluation with plain exponential gates, where the stabilizer
  of "The Stabilizer State: Preventing Numerical Overflow" (xLSTM Guide:
  Extended LSTM Architecture & Matrix Memory) must not change h;
* brute-force materialization of the causal decay matrix D of "The Dual
  Formulation: How mLSTM Enables Parallel GPU Training" (same guide), with the
  row normalizer |rowsum(D * Q K^T)| floored at 1;
* the closed form of the running-max stabilizer m_t;
* special cases that reduce to textbook formulas (normalized causal linear
  attention when nothing is forgotten; a memoryless cell when everything is);
* structural invariants (value columns, head order, which operand carries the
  1/sqrt(d) factor);
* hand-derived values for tiny inputs (tests/golden);
* planted mistakes: mutated copies of the oracle must fail these pins.
"""
from __future__ import annotations

import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def rand_case(rng, B=1, NH=2, S=12, dk=5, dv=3, ig=(0.0, 1.5), fg=(1.0, 2.0), kscale=1.0, og=True):
    f32 = np.float32
    q = rng.standard_normal((B, NH, S, dk)).astype(f32)
    k = (kscale * rng.standard_normal((B, NH, S, dk))).astype(f32)
    v = rng.standard_normal((B, NH, S, dv)).astype(f32)
    i = (ig[0] + ig[1] * rng.standard_normal((B, NH, S))).astype(f32)
    f = (fg[0] + fg[1] * rng.standard_normal((B, NH, S))).astype(f32)
    o = sigmoid(rng.standard_normal((B, NH, S, dv))).astype(f32) if og else None
    return q, k, v, i, f, o


# ---------------------------------------------------------------- independent forms


def closed_form(q, k, v, ig, fg, og):
    """Unrolled sums with explicit products of sigmoid forget gates (no recurrence)."""
    q, k, v, ig, fg = (np.asarray(x, np.float64) for x in (q, k, v, ig, fg))
    B, NH, S, dk = q.shape
    dv = v.shape[-1]
    h = np.zeros((B, NH, S, dv))
    Cbar = np.zeros((B, NH, dk, dv))
    nbar = np.zeros((B, NH, dk))
    for b in range(B):
        for hd in range(NH):
            f = sigmoid(fg[b, hd])
            for t in range(S):
                C = np.zeros((dk, dv))
                n = np.zeros(dk)
                for i in range(t + 1):
                    w = math.prod(f[j] for j in range(i + 1, t + 1)) * math.exp(ig[b, hd, i])
                    C += w * np.outer(k[b, hd, i], v[b, hd, i])
                    n += w * k[b, hd, i]
                qh = q[b, hd, t] / math.sqrt(dk)
                ht = C.T @ qh / max(abs(n @ qh), 1.0)
                if og is not None:
                    ht = ht * og[b, hd, t]
                h[b, hd, t] = ht
            Cbar[b, hd], nbar[b, hd] = C, n
    return h, Cbar, nbar


def unstabilized(q, k, v, ig, fg, og):
    """The recurrence with plain exponential gates and a denominator floor of 1."""
    q, k, v, ig, fg = (np.asarray(x, np.float64) for x in (q, k, v, ig, fg))
    B, NH, S, dk = q.shape
    dv = v.shape[-1]
    h = np.zeros((B, NH, S, dv))
    for b in range(B):
        for hd in range(NH):
            C = np.zeros((dk, dv))
            n = np.zeros(dk)
            for t in range(S):
                f = sigmoid(fg[b, hd, t])
                i = math.exp(ig[b, hd, t])
                C = f * C + i * np.outer(k[b, hd, t], v[b, hd, t])
                n = f * n + i * k[b, hd, t]
                qh = q[b, hd, t] / math.sqrt(dk)
                ht = C.T @ qh / max(abs(n @ qh), 1.0)
                h[b, hd, t] = ht * (og[b, hd, t] if og is not None else 1.0)
    return h


def dmatrix(q, k, v, ig, fg, og):
    """Full S x S causal decay matrix: log D_ij = sum_{l=j+1..i} log f_l + i~_j."""
    q, k, v, ig, fg = (np.asarray(x, np.float64) for x in (q, k, v, ig, fg))
    B, NH, S, dk = q.shape
    h = np.zeros(v.shape)
    for b in range(B):
        for hd in range(NH):
            logf = np.log(sigmoid(fg[b, hd]))
            logD = np.full((S, S), -np.inf)
            for i in range(S):
                for j in range(i + 1):
                    logD[i, j] = logf[j + 1:i + 1].sum() + ig[b, hd, j]
            D = np.exp(logD)
            Qh = q[b, hd] / math.sqrt(dk)
            W = D * (Qh @ k[b, hd].T)
            num = W @ v[b, hd]
            den = np.maximum(np.abs(W.sum(axis=1)), 1.0)[:, None]
            h[b, hd] = num / den * (og[b, hd] if og is not None else 1.0)
    return h


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


# ---------------------------------------------------------------- the pins as functions of a runner


def pin_closed_form(run, seed=0, **kw):
    rng = np.random.default_rng(seed)
    q, k, v, i, f, o = rand_case(rng, **kw)
    h, C, n, m = run(q, k, v, i, f, o)
    h_ref, Cbar, nbar = closed_form(q, k, v, i, f, o)
    scale = np.exp(m)[..., None]
    return max(rel(h, h_ref), rel(C * scale[..., None], Cbar), rel(n * scale, nbar))


def pin_unstabilized(run, seed=1, **kw):
    rng = np.random.default_rng(seed)
    q, k, v, i, f, o = rand_case(rng, **kw)
    h = run(q, k, v, i, f, o)[0]
    return rel(h, unstabilized(q, k, v, i, f, o))


def pin_dmatrix(run, seed=2, **kw):
    rng = np.random.default_rng(seed)
    q, k, v, i, f, o = rand_case(rng, **kw)
    h = run(q, k, v, i, f, o)[0]
    return rel(h, dmatrix(q, k, v, i, f, o))


def pin_m_closed_form(run, seed=3, m0=0.0, **kw):
    rng = np.random.default_rng(seed)
    q, k, v, i, f, o = rand_case(rng, **kw)
    B, NH, S, dk = q.shape
    dv = v.shape[-1]
    worst = 0.0
    m = np.full((B, NH), m0)
    C = np.zeros((B, NH, dk, dv))
    n = np.zeros((B, NH, dk))
    A = np.cumsum(np.log(sigmoid(f.astype(np.float64))), axis=-1)
    best = np.maximum.accumulate(i.astype(np.float64) - A, axis=-1)
    for t in range(S):
        _, C, n, m = run(q[:, :, t:t + 1], k[:, :, t:t + 1], v[:, :, t:t + 1], i[:, :, t:t + 1],
                         f[:, :, t:t + 1], None if o is None else o[:, :, t:t + 1], C, n, m)
        expect = A[..., t] + np.maximum(m0, best[..., t])
        worst = max(worst, float(np.max(np.abs(m - expect))))
    return worst


def all_pins(run):
    """Returns {pin name: error}; every value must be below its bound."""
    return {
        "closed_form": pin_closed_form(run),
        "closed_form_floor_binds": pin_closed_form(run, seed=10, kscale=0.02, ig=(-2.0, 2.0)),
        "closed_form_square": pin_closed_form(run, seed=11, dk=4, dv=4),
        "unstabilized": pin_unstabilized(run),
        "unstabilized_floor_binds": pin_unstabilized(run, seed=12, kscale=0.02, ig=(-3.0, 2.0)),
        "dmatrix": pin_dmatrix(run),
        "dmatrix_floor_binds": pin_dmatrix(run, seed=13, kscale=0.05, ig=(-2.0, 2.0)),
        "m_closed_form": pin_m_closed_form(run),
    }


PIN_BOUND = 1e-11


def oracle_run(q, k, v, i, f, o, C=None, n=None, m=None):
    return oracle.run(q, k, v, i, f, o, C, n, m)


# ---------------------------------------------------------------- tests


@pytest.mark.parametrize("name", ["closed_form", "closed_form_floor_binds", "closed_form_square",
                                  "unstabilized", "unstabilized_floor_binds", "dmatrix",
                                  "dmatrix_floor_binds", "m_closed_form"])
def test_pin(name):
    errs = all_pins(oracle_run)
    assert errs[name] < PIN_BOUND, errs


def test_floor_really_binds():
    """The floor cases above exercise the max(|n.q|, exp(-m)) branch on most rows."""
    rng = np.random.default_rng(10)
    q, k, v, i, f, o = rand_case(rng, kscale=0.02, ig=(-2.0, 2.0))
    _, Cbar, nbar = closed_form(q, k, v, i, f, o)
    qh = q[..., -1, :].astype(np.float64) / math.sqrt(q.shape[-1])
    assert np.all(np.abs((nbar * qh).sum(-1)) < 1.0)


@pytest.mark.parametrize("m0", [0.0, -np.inf, 5.0, -7.5])
def test_stabilizer_invariance(m0):
    """h does not depend on the initial stabilizer; e^m C and e^m n do not either."""
    rng = np.random.default_rng(4)
    q, k, v, i, f, o = rand_case(rng, S=16, ig=(0.0, 3.0))
    B, NH, S, dk = q.shape
    dv = v.shape[-1]
    h0, C0, n0, mm0 = oracle.run(q, k, v, i, f, o)
    h1, C1, n1, mm1 = oracle.run(q, k, v, i, f, o, np.zeros((B, NH, dk, dv)), np.zeros((B, NH, dk)),
                                 np.full((B, NH), m0))
    assert rel(h1, h0) < 1e-13
    assert rel(C1 * np.exp(mm1)[..., None, None], C0 * np.exp(mm0)[..., None, None]) < 1e-13
    assert rel(n1 * np.exp(mm1)[..., None], n0 * np.exp(mm0)[..., None]) < 1e-13


@pytest.mark.parametrize("m0", [0.0, 2.5, -4.0])
def test_m_closed_form_from_state(m0):
    assert pin_m_closed_form(oracle_run, seed=5, m0=m0) < 1e-12


def test_linear_attention_limit():
    """No forgetting and unit input gates: normalized causal linear attention."""
    rng = np.random.default_rng(6)
    q, k, v, i, f, o = rand_case(rng, S=20, og=False)
    i[:] = 0.0
    f[:] = 1e4                      # logsigmoid(1e4) == 0 in double precision
    h = oracle.run(q, k, v, i, f, None)[0]
    qd, kd, vd = (x.astype(np.float64) for x in (q, k, v))
    dk = q.shape[-1]
    ref = np.zeros_like(h)
    for b in range(q.shape[0]):
        for hd in range(q.shape[1]):
            A = (qd[b, hd] / math.sqrt(dk)) @ kd[b, hd].T
            A = np.tril(A)
            ref[b, hd] = (A @ vd[b, hd]) / np.maximum(np.abs(A.sum(1)), 1.0)[:, None]
    assert rel(h, ref) < 1e-12


@pytest.mark.parametrize("S", [1, 9])
def test_memoryless_limit(S):
    """Everything forgotten (and S = 1): h_t = o v_t (qh.k_t) / max(|qh.k_t|, exp(-i~_t))."""
    rng = np.random.default_rng(7)
    q, k, v, i, f, o = rand_case(rng, S=S, ig=(0.0, 3.0))
    if S > 1:
        f[:] = -1e4
    h = oracle.run(q, k, v, i, f, o)[0]
    dk = q.shape[-1]
    s = (q.astype(np.float64) * k).sum(-1) / math.sqrt(dk)
    ref = o.astype(np.float64) * v.astype(np.float64) * (s / np.maximum(np.abs(s), np.exp(-i.astype(np.float64))))[..., None]
    assert rel(h, ref) < 1e-12


def test_value_columns_independent():
    """Column j of h and of C depends only on column j of v and o."""
    rng = np.random.default_rng(8)
    q, k, v, i, f, o = rand_case(rng, dv=7)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    cols = [5, 1, 3]
    h2, C2, n2, m2 = oracle.run(q, k, v[..., cols], i, f, o[..., cols])
    assert rel(h2, h[..., cols]) < 1e-14 and rel(C2, C[..., cols]) < 1e-14
    assert rel(n2, n) == 0.0 and rel(m2, m) == 0.0


def test_heads_independent():
    rng = np.random.default_rng(9)
    q, k, v, i, f, o = rand_case(rng, B=2, NH=3)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    perm = [2, 0, 1]
    h2, C2, n2, m2 = oracle.run(q[:, perm], k[:, perm], v[:, perm], i[:, perm], f[:, perm], o[:, perm])
    assert np.array_equal(h2, h[:, perm]) and np.array_equal(C2, C[:, perm])
    assert np.array_equal(n2, n[:, perm]) and np.array_equal(m2, m[:, perm])


def test_scaling_k_instead_of_q():
    """Moving the 1/sqrt(d) factor from q to k leaves h unchanged and scales C, n by it."""
    rng = np.random.default_rng(14)
    q, k, v, i, f, o = rand_case(rng, dk=16, kscale=0.1)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    h2, C2, n2, m2 = oracle.run(q * np.float32(4.0), k / np.float32(4.0), v, i, f, o)
    assert rel(h2, h) < 1e-13 and rel(C2 * 4.0, C) < 1e-13 and rel(n2 * 4.0, n) < 1e-13


def test_split_sequence_equals_whole():
    """Running S tokens equals running S1 tokens, then S - S1 more from that state."""
    rng = np.random.default_rng(15)
    q, k, v, i, f, o = rand_case(rng, S=13)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    s1 = 5
    ha, Ca, na, ma = oracle.run(q[:, :, :s1], k[:, :, :s1], v[:, :, :s1], i[:, :, :s1], f[:, :, :s1],
                                o[:, :, :s1])
    hb, Cb, nb, mb = oracle.run(q[:, :, s1:], k[:, :, s1:], v[:, :, s1:], i[:, :, s1:], f[:, :, s1:],
                                o[:, :, s1:], Ca, na, ma)
    assert np.array_equal(np.concatenate([ha, hb], axis=2), h)
    assert np.array_equal(Cb, C) and np.array_equal(mb, m)


def test_step_is_one_token_run():
    rng = np.random.default_rng(16)
    q, k, v, i, f, o = rand_case(rng, S=6)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    hs, Cs, ns, ms = oracle.run(q[:, :, :5], k[:, :, :5], v[:, :, :5], i[:, :, :5], f[:, :, :5], o[:, :, :5])
    h1, C1, n1, m1 = oracle.mlstm_step(Cs, ns, ms, q[:, :, 5], k[:, :, 5], v[:, :, 5], i[:, :, 5], f[:, :, 5],
                                       o[:, :, 5])
    assert np.array_equal(h1, h[:, :, 5]) and np.array_equal(C1, C) and np.array_equal(m1, m)


def test_empty_sequence_keeps_state():
    rng = np.random.default_rng(17)
    q, k, v, i, f, o = rand_case(rng, S=0)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    assert h.shape[2] == 0 and not C.any() and not n.any() and not m.any()


@pytest.mark.parametrize("fname", sorted(x for x in os.listdir(GOLDEN) if x.startswith("hand_")))
def test_hand_derived(fname):
    """Values worked out by hand from the recurrence (derivations in the fixture)."""
    g = json.load(open(os.path.join(GOLDEN, fname)))
    dk, dv = g["DHQK"], g["DHV"]
    S = len(g["igate"])
    arr = lambda key, d: np.array(g[key], dtype=np.float32).reshape(1, 1, S, d)
    q, k, v = arr("q", dk), arr("k", dk), arr("v", dv)
    o = arr("o", dv) if g.get("o") is not None else None
    i = np.array(g["igate"], dtype=np.float32).reshape(1, 1, S)
    f = np.array(g["fgate"], dtype=np.float32).reshape(1, 1, S)
    h, C, n, m = oracle.run(q, k, v, i, f, o)
    tol = g["tolerance"]
    np.testing.assert_allclose(h.reshape(S, dv), np.array(g["h"], dtype=np.float64).reshape(S, dv),
                               rtol=tol, atol=tol)
    np.testing.assert_allclose(C.reshape(dk, dv), np.array(g["C_final"]).reshape(dk, dv), rtol=tol, atol=tol)
    np.testing.assert_allclose(n.reshape(dk), np.array(g["n_final"]), rtol=tol, atol=tol)
    np.testing.assert_allclose(m.reshape(1), np.array([g["m_final"]]), rtol=tol, atol=tol)


# ---------------------------------------------------------------- planted mistakes

MUTATIONS = {
    "floor_sign": ("exp(-m_new)", "exp(m_new)"),
    "no_q_scale": ("(double)qt[i] * scale", "(double)qt[i]"),
    "forget_uses_new_m": ("exp(lf + m_prev - m_new)", "exp(lf + m_new - m_new)"),
    "raw_forget_gate": ("const double lf = log_sigmoid((double)fg[t]);", "const double lf = (double)fg[t];"),
    "normalizer_drops_input": ("n[i] = fp * n[i] + ip * kt[i];", "n[i] = fp * n[i] + kt[i];"),
    "readout_before_decay": ("row[j] = fp * row[j] + ik * vt[j];", "row[j] = row[j] + ik * vt[j];"),
    "transposed_memory": ("ht[j] += qi * row[j];", "ht[j] += qh[j % dk] * C[(size_t)(j % dk) * dv + i % dv];"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("mutants")


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, mutant_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mlstm_oracle.c")).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) == 1, "mutation anchor not found: %s" % old
    path_c = os.path.join(mutant_dir, mutation + ".c")
    path_so = os.path.join(mutant_dir, mutation + ".so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", path_so, path_c, "-lm",
                           "-lpthread"])
    lib = oracle.load_library(path_so)

    def run(q, k, v, i, f, o, C=None, n=None, m=None):
        return oracle.run(q, k, v, i, f, o, C, n, m, lib=lib)

    errs = all_pins(run)
    assert max(errs.values()) > 1e-6, errs
