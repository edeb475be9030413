"""Pins of the C adjoint gradient oracle (oracle/mlstm_adjoint.c).

The adjoint is reverse-mode differentiation of the recurrence written out by hand, token by token;
it is checked against torch.autograd's derivatives of the same recurrence (oracle/mlstm_bwd.py,
itself pinned by finite differences, the output-gate identity and the dual-form value gradient)
on shapes that make the denominator floor inactive and binding, with adversarial gates, with and
without an output gate, and at token counts that cross several checkpoint segments.  Planted
mistakes in copies of the adjoint must fail that check.
"""
from __future__ import annotations

import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import mlstm_bwd

NAMES = ("dq", "dk", "dv", "digate", "dfgate", "dogate")


def _inputs(B, NH, S, dk, dv, seed, scale=1.0, ig=(0.0, 1.0), fg=(2.0, 1.0), ogate=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, NH, S, dk, generator=g) * scale
    k = torch.randn(B, NH, S, dk, generator=g) * scale
    v = torch.randn(B, NH, S, dv, generator=g)
    i = torch.randn(B, NH, S, generator=g) * ig[1] + ig[0]
    f = torch.randn(B, NH, S, generator=g) * fg[1] + fg[0]
    o = torch.sigmoid(torch.randn(B, NH, S, dv, generator=g)) if ogate else None
    dh = torch.randn(B, NH, S, dv, generator=g)
    return q, k, v, i, f, o, dh   # float32: both oracles see the same numbers


CASES = [
    dict(B=1, NH=2, S=23, dk=5, dv=4, seed=1),
    dict(B=2, NH=1, S=40, dk=8, dv=6, seed=2, scale=0.02),                # denominator floor binds
    dict(B=1, NH=2, S=31, dk=4, dv=3, seed=3, ig=(0.0, 8.0)),             # dominant tokens
    dict(B=1, NH=1, S=29, dk=6, dv=5, seed=4, fg=(-4.0, 1.0)),            # fast forgetting
    dict(B=1, NH=1, S=50, dk=4, dv=4, seed=5, ogate=False),
    dict(B=1, NH=1, S=1, dk=3, dv=2, seed=6),
]


def _max_rel(got, ref):
    errs = {}
    for name, x, r in zip(NAMES, got, ref):
        if r is None:
            assert x is None
            continue
        # relative error, against an absolute floor for gradients that are exactly zero in real
        # arithmetic (one token whose denominator does not bind: h does not depend on its i~)
        errs[name] = float(np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-3))
    return errs


def _autograd(q, k, v, i, f, o, dh):
    return mlstm_bwd.mlstm_bwd(q.double(), k.double(), v.double(), i.double(), f.double(),
                               None if o is None else o.double(), dh.double())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "S%d_d%dx%d_seed%d" % (c["S"], c["dk"], c["dv"], c["seed"]))
def test_adjoint_equals_autograd(case):
    xs = _inputs(**case)
    got = oracle.mlstm_adjoint(*xs, nthreads=2)
    errs = _max_rel(got, _autograd(*xs))
    assert max(errs.values()) <= 1e-11, errs


def test_heads_are_independent():
    xs = _inputs(B=2, NH=2, S=17, dk=4, dv=3, seed=9)
    whole = oracle.mlstm_adjoint(*xs)
    one = oracle.mlstm_adjoint(*[None if x is None else x[1:2, 0:1] for x in xs])
    for a, b in zip(whole, one):
        np.testing.assert_allclose(a[1:2, 0:1], b, rtol=1e-13, atol=0)


MUTATIONS = {
    "no_q_scale_in_dq": ("H->dq[(size_t)t * dk + i] = (a + dden * nt[i]) * scale;",
                         "H->dq[(size_t)t * dk + i] = (a + dden * nt[i]);"),
    "floor_branch_ignored": ("const double dden = fabs(den) > floor_ ? (den > 0.0 ? dN : -dN) : 0.0;",
                             "const double dden = den > 0.0 ? dN : -dN;"),
    "state_gradient_not_decayed": ("dC[e] *= fp;", "dC[e] *= 1.0;"),
    "forget_without_sigmoid_factor": ("H->dfg[t] = fp * dfp * sigmoid(-(double)H->fg[t]);",
                                      "H->dfg[t] = fp * dfp;"),
    "input_gate_without_weight": ("H->dig[t] = ip * dip;", "H->dig[t] = dip;"),
    "value_gradient_transposed": ("a += dC[(size_t)i * dv + jj] * (double)kt[i];",
                                  "a += dC[(size_t)(jj % dk) * dv + i % dv] * (double)kt[i];"),
    "normalizer_gradient_dropped": ("dCv[i] = a + dn[i];", "dCv[i] = a;"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("adjoint_mutants")


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, mutant_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "mlstm_adjoint.c")).read()
    old, new = MUTATIONS[mutation]
    assert src.count(old) == 1, "mutation anchor not found: %s" % old
    path_c = os.path.join(mutant_dir, mutation + ".c")
    path_so = os.path.join(mutant_dir, mutation + ".so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", path_so, path_c, "-lm", "-lpthread"])
    lib = oracle.load_adjoint_library(path_so)
    worst = 0.0
    for case in CASES:
        xs = _inputs(**case)
        errs = _max_rel(oracle.mlstm_adjoint(*xs, nthreads=2, lib=lib), _autograd(*xs))
        worst = max(worst, max(errs.values()))
    assert worst > 1e-6, worst
