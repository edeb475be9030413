"""fp64 CPU oracle of the mLSTM cell (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library and its binding never do.  The arithmetic lives
in ``mlstm_oracle.c`` (plain C, double precision, one head at a time, token by
token); this module compiles it with gcc and marshals numpy arrays.

Two more modules live beside it, for the library's other entry points: ``oracle.slstm`` (the
sLSTM cell's recurrence, numpy float64) and ``oracle.mlstm_bwd`` (gradients of the forward pass,
float64 torch autograd of the plain recurrence).

Layouts follow the library: q, k ``[B, NH, T, DHQK]``; v, o ``[B, NH, T, DHV]``;
gates ``[B, NH, T]``; state C ``[B, NH, DHQK, DHV]``, n ``[B, NH, DHQK]``,
m ``[B, NH]``.  Inputs are converted to float32 (exact for fp32 and bf16
data); outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlstm_oracle.c")
_LIB = os.path.join(_HERE, "libmlstm_oracle.so")
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc (IEEE double, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Loads an oracle shared library built from ``mlstm_oracle.c`` (or a variant of it)."""
    lib = ctypes.CDLL(path)
    lib.oracle_mlstm_run.restype = ctypes.c_int
    lib.oracle_mlstm_run.argtypes = [ctypes.c_int] * 4 + [_f32p] * 6 + [_f64p] * 4 + [ctypes.c_int]
    lib.oracle_default_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _f32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor: widen on the CPU (bf16 -> fp32 is exact)
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def run(q, k, v, igate, fgate, ogate=None, C=None, n=None, m=None,
        want_h: bool = True, nthreads: int = 0, lib=None, inplace: bool = False):
    """Runs the recurrence over the T tokens of the inputs from state (C, n, m).

    A missing state is the zero state (C = 0, n = 0, m = 0).  Returns
    ``(h, C, n, m)`` in float64 (h is None when ``want_h`` is False).  With
    ``inplace`` the given state arrays (float64, C-contiguous numpy) are updated
    in place and returned instead of copied first (large decode states).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    ig, fg, og = _f32(igate), _f32(fgate), _f32(ogate)
    B, NH, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, NH, T, dk) and v.shape == (B, NH, T, dv)
    assert ig.shape == (B, NH, T) and fg.shape == (B, NH, T)
    assert og is None or og.shape == (B, NH, T, dv)
    def state(x, shape):
        if x is None:
            return np.zeros(shape)
        if inplace:
            assert isinstance(x, np.ndarray) and x.dtype == np.float64 and x.flags["C_CONTIGUOUS"]
            return x
        return np.array(x, dtype=np.float64, order="C")
    Cs, ns, ms = state(C, (B, NH, dk, dv)), state(n, (B, NH, dk)), state(m, (B, NH))
    assert Cs.shape == (B, NH, dk, dv) and ns.shape == (B, NH, dk) and ms.shape == (B, NH)
    h = np.empty((B, NH, T, dv)) if want_h else None
    rc = (lib or _load()).oracle_mlstm_run(B * NH, T, dk, dv, _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p),
                                  _ptr(ig, _f32p), _ptr(fg, _f32p), _ptr(og, _f32p),
                                  _ptr(Cs, _f64p), _ptr(ns, _f64p), _ptr(ms, _f64p),
                                  _ptr(h, _f64p), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mlstm_run rejected its arguments")
    return h, Cs, ns, ms


def mlstm_fwd(q, k, v, igate, fgate, ogate=None, nthreads: int = 0):
    """Forward pass from the zero state: ``(h, C_final, n_final, m_final)``."""
    return run(q, k, v, igate, fgate, ogate, nthreads=nthreads)


def mlstm_step(C, n, m, q, k, v, igate, fgate, ogate=None, nthreads: int = 0, inplace: bool = False):
    """One decode step on a state; token inputs are ``[B, NH, D]`` and ``[B, NH]``.

    Returns ``(h [B, NH, DHV], C', n', m')`` (with ``inplace``, the given float64 state arrays,
    updated).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    og = _f32(ogate)
    h, C2, n2, m2 = run(q[:, :, None], k[:, :, None], v[:, :, None],
                        _f32(igate)[:, :, None], _f32(fgate)[:, :, None],
                        None if og is None else og[:, :, None], C, n, m, nthreads=nthreads, inplace=inplace)
    return h[:, :, 0], C2, n2, m2
