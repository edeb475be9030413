"""Helpers shared by the GPU parity tests: error metric and tolerances.

The error of an output is its relative L2 error against the fp64 oracle over the
whole tensor, ||x - x_ref||_2 / ||x_ref||_2, taken separately for h, C, n and m.
Limits: 1e-5 when q, k, v are float32 and 1e-2 when they are bf16 (states and
accumulation are float32 in both cases).
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {"f32": 1e-5, "bf16": 1e-2}


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rel_l2(x, ref) -> float:
    x, ref = to64(x), to64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    d = np.linalg.norm((x - ref).ravel())
    n = np.linalg.norm(ref.ravel())
    if n == 0.0:
        return float(d)
    return float(d / n)


def assert_close(name: str, x, ref, tol: float):
    err = rel_l2(x, ref)
    assert np.all(np.isfinite(to64(x))), "%s has non-finite values" % name
    assert err <= tol, "%s: rel-L2 %.3e > %.1e" % (name, err, tol)
    return err


class L2Acc:
    """Relative L2 error of a tensor compared piece by piece (sum of squared differences and of
    squared reference values over the pieces), for outputs too large to hold twice in fp64."""

    def __init__(self):
        self.diff = 0.0
        self.ref = 0.0

    def add(self, x, ref):
        x, ref = to64(x), to64(ref)
        assert x.shape == ref.shape, (x.shape, ref.shape)
        assert np.all(np.isfinite(x)), "non-finite values"
        self.diff += float(np.sum(np.square(x - ref)))
        self.ref += float(np.sum(np.square(ref)))

    def rel(self) -> float:
        return float(np.sqrt(self.diff) / np.sqrt(self.ref)) if self.ref > 0 else float(np.sqrt(self.diff))
