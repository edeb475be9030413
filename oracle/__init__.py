"""fp64 CPU oracle of the mLSTM cell (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library and its binding never do.  The arithmetic lives
in ``mlstm_oracle.c`` (plain C, double precision, one head at a time, token by
token); this module compiles it with gcc and marshals numpy arrays.

Beside it, for the library's other entry points: ``oracle.slstm`` (the sLSTM cell's recurrence,
numpy float64), ``oracle.mlstm_bwd`` (gradients of the forward pass, float64 torch autograd of the
plain recurrence) and ``mlstm_adjoint.c`` / ``mlstm_adjoint()`` (the same gradients by the
token-by-token adjoint of the recurrence written out in C, fast enough for full-size shapes; pinned
against the autograd gradients).

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
_ADJ_SRC = os.path.join(_HERE, "mlstm_adjoint.c")
_ADJ_LIB = os.path.join(_HERE, "libmlstm_adjoint.so")
_lib = None
_adj_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


def _gcc(src: str, lib: str, force: bool) -> str:
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        tmp = lib + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-ffp-contract=off", "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compiles the oracle (and the gradient adjoint) with gcc (IEEE double, no fast-math) if stale."""
    _gcc(_ADJ_SRC, _ADJ_LIB, force)
    return _gcc(_SRC, _LIB, force)


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


def load_adjoint_library(path: str):
    """Loads a gradient library built from ``mlstm_adjoint.c`` (or a variant of it)."""
    lib = ctypes.CDLL(path)
    lib.oracle_mlstm_adjoint.restype = ctypes.c_int
    lib.oracle_mlstm_adjoint.argtypes = [ctypes.c_int] * 4 + [_f32p] * 7 + [_f64p] * 6 + [ctypes.c_int]
    return lib


def mlstm_adjoint(q, k, v, igate, fgate, ogate, dh, nthreads: int = 0, lib=None):
    """Gradients of sum(dh * h) of the forward pass from the zero state, by the token-by-token
    adjoint of the recurrence in ``mlstm_adjoint.c``: ``(dq, dk, dv, digate, dfgate, dogate)`` in
    float64 (dogate None without an output gate)."""
    global _adj_lib
    if lib is None:
        if _adj_lib is None:
            build()
            _adj_lib = load_adjoint_library(_ADJ_LIB)
        lib = _adj_lib
    q, k, v, dh = _f32(q), _f32(k), _f32(v), _f32(dh)
    ig, fg, og = _f32(igate), _f32(fgate), _f32(ogate)
    B, NH, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape == (B, NH, T, dv) and dh.shape == v.shape
    assert ig.shape == (B, NH, T) and fg.shape == (B, NH, T) and (og is None or og.shape == v.shape)
    dq, dkk = np.empty(q.shape), np.empty(q.shape)
    dvv = np.empty(v.shape)
    dig, dfg = np.empty(ig.shape), np.empty(ig.shape)
    dog = np.empty(v.shape) if og is not None else None
    rc = lib.oracle_mlstm_adjoint(B * NH, T, dk, dv, _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p),
                                  _ptr(ig, _f32p), _ptr(fg, _f32p), _ptr(og, _f32p), _ptr(dh, _f32p),
                                  _ptr(dq, _f64p), _ptr(dkk, _f64p), _ptr(dvv, _f64p), _ptr(dig, _f64p),
                                  _ptr(dfg, _f64p), _ptr(dog, _f64p), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mlstm_adjoint rejected its arguments")
    return dq, dkk, dvv, dig, dfg, dog
