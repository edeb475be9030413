"""Thin ctypes binding of libmlstm (argument marshalling only).

The functions take torch tensors that already live on the GPU, pass their
device pointers, sizes and the current CUDA stream to the C ABI declared in
``include/mlstm.h``, and raise ``MlstmError`` on a non-zero status.  Every step
of the computation runs in the library's CUDA kernels; there is no other code
path.  If the library cannot be loaded the import of the functions fails
loudly (``load()`` raises).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmlstm.so")

MLSTM_F32, MLSTM_BF16 = 0, 1
STATUS = {0: "MLSTM_OK", 1: "MLSTM_ERR_INVALID_ARG", 2: "MLSTM_ERR_UNSUPPORTED", 3: "MLSTM_ERR_WORKSPACE",
          4: "MLSTM_ERR_CUDA", 5: "MLSTM_ERR_TIMEOUT"}

# Every symbol include/mlstm.h and include/slstm.h declare, with its ctypes signature.
_vp, _fp, _i, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "mlstm_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "mlstm_fwd": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _fp, _fp, _fp, _vp, _sz,
                       _vp]),
    "mlstm_fwd_state": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp, _fp, _fp,
                             _fp, _vp, _sz, _vp]),
    "mlstm_fwd_profiled": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _fp, _fp, _fp,
                                _vp, _sz, _vp, ctypes.POINTER(ctypes.c_void_p)]),
    "mlstm_fwd_status": (_i, [_vp, _vp]),
    "mlstm_fwd_noalloc": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _fp, _fp, _fp,
                               _vp]),
    "mlstm_fwd_noalloc_status": (_i, [_vp]),
    "mlstm_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "mlstm_bwd": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _fp, _fp, _vp,
                       _vp, _sz, _vp]),
    "mlstm_fwd_kernel_launches": (_i, [_i, _i, _i, _i, _i, _i, _i]),
    "mlstm_fwd_tensor_path": (_i, [_i, _i, _i, _i]),
    "mlstm_fwd_paired_walk": (_i, [_i, _i, _i, _i]),
    "mlstm_bwd_tensor_path": (_i, [_i, _i, _i, _i]),
    "mlstm_fwd_segments": (_i, [_i, _i, _i, _i, _i, _i, _i]),
    "mlstm_step": (_i, [_fp, _fp, _fp, _vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "mlstm_status_string": (ctypes.c_char_p, [_i]),
    "mlstm_fwd_final_state": (_i, [_vp, _vp, _fp, _fp, _i, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp, _sz, _vp]),
    "mlstm_log_decay_sum": (_i, [_fp, _i, _i, _i, _fp, _vp]),
    "mlstm_state_prefix": (_i, [_fp, _fp, _fp, _fp, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _vp]),
    "mlstm_selftest_wait_timeout": (_i, [_vp, _vp]),
    "slstm_fwd": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _fp, _fp, _fp, _fp, _vp, _vp, _vp]),
    "slstm_batch_per_cluster": (_i, [_i, _i, _i, _i]),
}

_lib = None


class MlstmError(RuntimeError):
    def __init__(self, fn: str, status: int, lib=None):
        text = lib.mlstm_status_string(status).decode() if lib is not None else ""
        super().__init__("%s returned %s (%s)" % (fn, STATUS.get(status, status), text))
        self.status = status


def load(path: str | None = None):
    """Loads libmlstm.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError("libmlstm.so not found at %s; build it with `python -m xlstm_mlstm_cell_b200.build`" % p)
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MLSTM_F32
    if t.dtype == torch.bfloat16:
        return MLSTM_BF16
    raise TypeError("q, k, v must be float32 or bfloat16, got %s" % t.dtype)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise MlstmError(fn, status, _lib)


def workspace_size(B, NH, S, DHQK, DHV, chunk, dtype) -> int:
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_fwd_workspace_size(B, NH, S, DHQK, DHV, chunk, dt))


def fwd_kernel_launches(B, NH, S, DHQK, DHV, chunk, dtype) -> int:
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_fwd_kernel_launches(B, NH, S, DHQK, DHV, chunk, dt))


def fwd_tensor_path(DHQK, DHV, chunk, dtype) -> int:
    """1: tensor-core path, 0: fp32 CUDA-core path, -1: unsupported (mlstm_fwd_tensor_path)."""
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_fwd_tensor_path(DHQK, DHV, chunk, dt))


def fwd_paired_walk(DHQK, DHV, chunk, dtype) -> int:
    """1: the walk runs as CTA pairs, 0: one CTA per value tile, -1: off the tensor-core path
    (mlstm_fwd_paired_walk)."""
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_fwd_paired_walk(DHQK, DHV, chunk, dt))


def fwd_segments(B, NH, S, DHQK, DHV, chunk, dtype) -> int:
    """Segments per head of the tensor-core path for this shape (0 off that path)."""
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_fwd_segments(B, NH, S, DHQK, DHV, chunk, dt))


def alloc_workspace(B, NH, S, DHQK, DHV, chunk, dtype, device="cuda") -> torch.Tensor:
    n = workspace_size(B, NH, S, DHQK, DHV, chunk, dtype)
    if n == 0:
        raise MlstmError("mlstm_fwd_workspace_size", 2)
    return torch.empty(n, dtype=torch.uint8, device=device)


FWD_PHASES = 4
PHASE_NAMES = ("gate_prep", "state_contributions", "state_scan", "outputs")


def fwd(q, k, v, igate, fgate, ogate=None, chunk: int = 64, h_out=None, C_final=None, n_final=None,
        m_final=None, workspace=None, return_state: bool = True, stream=None, events=None, state=None):
    """mlstm_fwd on device tensors; returns ``(h, C, n, m)`` (states None unless requested).

    ``state=(C0, n0, m0)`` starts from that state (mlstm_fwd_state) instead of the zero state.
    With ``events`` (FWD_PHASES + 1 ``torch.cuda.Event`` or None) the call goes through
    mlstm_fwd_profiled, which records them around its phases on the stream; ``events[FWD_PHASES
    - 1]`` completes once the final state is written.
    """
    lib = load()
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    dt = _dt(q)
    if h_out is None:
        h_out = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=q.device)
    if return_state:
        if C_final is None:
            C_final = torch.empty((B, NH, DHQK, DHV), dtype=torch.float32, device=q.device)
        if n_final is None:
            n_final = torch.empty((B, NH, DHQK), dtype=torch.float32, device=q.device)
        if m_final is None:
            m_final = torch.empty((B, NH), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, NH, S, DHQK, DHV, chunk, q.dtype, q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate), dt, B, NH, S, DHQK, DHV, chunk,
            _ptr(h_out), _ptr(C_final), _ptr(n_final), _ptr(m_final), _ptr(workspace), workspace.numel(),
            _stream(stream))
    if state is not None:
        assert events is None
        C0, n0, m0 = state
        sargs = args[:13] + (_ptr(C0), _ptr(n0), _ptr(m0)) + args[13:]
        _check("mlstm_fwd_state", lib.mlstm_fwd_state(*sargs))
    elif events is None:
        _check("mlstm_fwd", lib.mlstm_fwd(*args))
    else:
        assert len(events) == FWD_PHASES + 1
        for e in events:            # torch creates the CUDA event lazily, on its first record
            if e is not None and not e.cuda_event:
                e.record()
        arr = (ctypes.c_void_p * (FWD_PHASES + 1))(*[None if e is None else e.cuda_event for e in events])
        _check("mlstm_fwd_profiled", lib.mlstm_fwd_profiled(*args, arr))
    return h_out, C_final, n_final, m_final


def bwd_tensor_path(DHQK, DHV, chunk, dtype) -> int:
    """mlstm_bwd_tensor_path: 1 for the tensor-core gradient products, 0 for the CUDA cores, -1 unsupported."""
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_bwd_tensor_path(DHQK, DHV, chunk, dt))


def bwd_workspace_size(B, NH, S, DHQK, DHV, chunk, dtype) -> int:
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().mlstm_bwd_workspace_size(B, NH, S, DHQK, DHV, chunk, dt))


def bwd(q, k, v, igate, fgate, ogate, dh, chunk: int = 64, workspace=None, stream=None, out=None):
    """mlstm_bwd on device tensors: gradients of sum(dh * h) for the forward pass from the zero
    state.  Returns ``(dq, dk, dv, digate, dfgate, dogate)`` (dogate None without an output gate);
    ``out`` may give those six tensors to write into."""
    lib = load()
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    dt = _dt(q)
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(igate),
               torch.empty_like(fgate), None if ogate is None else torch.empty_like(ogate))
    dq, dk, dv, dig, dfg, dog = out
    if workspace is None:
        n = bwd_workspace_size(B, NH, S, DHQK, DHV, chunk, q.dtype)
        if n == 0:
            raise MlstmError("mlstm_bwd_workspace_size", 2)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    _check("mlstm_bwd", lib.mlstm_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate), _ptr(dh), dt,
                                      B, NH, S, DHQK, DHV, chunk, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dig), _ptr(dfg),
                                      _ptr(dog), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv, dig, dfg, dog


def fwd_final_state(k, v, igate, fgate, chunk: int = 64, workspace=None, stream=None):
    """mlstm_fwd_final_state: ``(C, n, m)`` of the sequence from the zero state, no outputs."""
    lib = load()
    B, NH, S, DHQK = k.shape
    DHV = v.shape[-1]
    C = torch.empty((B, NH, DHQK, DHV), dtype=torch.float32, device=k.device)
    n = torch.empty((B, NH, DHQK), dtype=torch.float32, device=k.device)
    m = torch.empty((B, NH), dtype=torch.float32, device=k.device)
    if workspace is None:
        workspace = alloc_workspace(B, NH, S, DHQK, DHV, chunk, k.dtype, k.device)
    _check("mlstm_fwd_final_state",
           lib.mlstm_fwd_final_state(_ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _dt(k), B, NH, S, DHQK, DHV, chunk,
                                     _ptr(C), _ptr(n), _ptr(m), _ptr(workspace), workspace.numel(), _stream(stream)))
    return C, n, m


def log_decay_sum(fgate, stream=None):
    """mlstm_log_decay_sum: per (b, h) the sum over tokens of logsigmoid(f~), ``[B, NH]``."""
    lib = load()
    B, NH, S = fgate.shape
    g = torch.empty((B, NH), dtype=torch.float32, device=fgate.device)
    _check("mlstm_log_decay_sum", lib.mlstm_log_decay_sum(_ptr(fgate), B, NH, S, _ptr(g), _stream(stream)))
    return g


def state_prefix(C_parts, n_parts, m_parts, g_parts, rank: int, stream=None):
    """mlstm_state_prefix: the start state ``(C0, n0, m0)`` of slice ``rank`` from the gathered
    summaries ``C_parts [R, B, NH, DHQK, DHV]``, ``n_parts [R, B, NH, DHQK]``, ``m_parts`` and
    ``g_parts [R, B, NH]``."""
    lib = load()
    R, B, NH, DHQK, DHV = C_parts.shape
    C0 = torch.empty((B, NH, DHQK, DHV), dtype=torch.float32, device=C_parts.device)
    n0 = torch.empty((B, NH, DHQK), dtype=torch.float32, device=C_parts.device)
    m0 = torch.empty((B, NH), dtype=torch.float32, device=C_parts.device)
    _check("mlstm_state_prefix",
           lib.mlstm_state_prefix(_ptr(C_parts), _ptr(n_parts), _ptr(m_parts), _ptr(g_parts), R, rank, B, NH, DHQK,
                                  DHV, _ptr(C0), _ptr(n0), _ptr(m0), _stream(stream)))
    return C0, n0, m0


NOALLOC_MAX_BYTES = 32 * 1024 * 1024


def fwd_noalloc(q, k, v, igate, fgate, ogate=None, chunk: int = 64, h_out=None, C_final=None, n_final=None,
                m_final=None, stream=None):
    """mlstm_fwd_noalloc: the forward pass with the library's built-in scratch array.

    For callers that may not allocate device memory for a workspace (the outputs are still
    the caller's).  Returns ``(h, C, n, m)``.
    """
    lib = load()
    B, NH, S, DHQK = q.shape
    DHV = v.shape[-1]
    if h_out is None:
        h_out = torch.empty((B, NH, S, DHV), dtype=q.dtype, device=q.device)
    if C_final is None:
        C_final = torch.empty((B, NH, DHQK, DHV), dtype=torch.float32, device=q.device)
    if n_final is None:
        n_final = torch.empty((B, NH, DHQK), dtype=torch.float32, device=q.device)
    if m_final is None:
        m_final = torch.empty((B, NH), dtype=torch.float32, device=q.device)
    st = lib.mlstm_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate), _ptr(ogate), _dt(q), B, NH,
                               S, DHQK, DHV, chunk, _ptr(h_out), _ptr(C_final), _ptr(n_final), _ptr(m_final),
                               _stream(stream))
    _check("mlstm_fwd_noalloc", st)
    return h_out, C_final, n_final, m_final


def fwd_noalloc_status(stream=None) -> int:
    """mlstm_fwd_noalloc_status: 0 when the last mlstm_fwd_noalloc on this device completed, else the
    status code (MLSTM_ERR_TIMEOUT after a bounded wait gave up); synchronizes the stream."""
    return int(load().mlstm_fwd_noalloc_status(_stream(stream)))


def fwd_status(workspace, stream=None) -> int:
    return int(load().mlstm_fwd_status(_ptr(workspace), _stream(stream)))


def step(C, n, m, q, k, v, igate, fgate, ogate=None, h_out=None, stream=None):
    """mlstm_step on device tensors; the state (C, n, m) is updated in place; returns h."""
    lib = load()
    B, NH, DHQK = q.shape
    DHV = v.shape[-1]
    if h_out is None:
        h_out = torch.empty((B, NH, DHV), dtype=q.dtype, device=q.device)
    st = lib.mlstm_step(_ptr(C), _ptr(n), _ptr(m), _ptr(q), _ptr(k), _ptr(v), _ptr(igate), _ptr(fgate),
                        _ptr(ogate), _dt(q), B, NH, DHQK, DHV, _ptr(h_out), _stream(stream))
    _check("mlstm_step", st)
    return h_out


def slstm_fwd(wx, R, forget: str = "exp", state=None, h_out=None, want_h: bool = True, status=None, stream=None):
    """slstm_fwd on device tensors: S steps of the sLSTM recurrence.

    wx [B, S, 4, NH, DH] gate pre-activations (i, f, z, o), R [NH, 4, DH, DH], both float32 or
    bfloat16; forget "exp" or "sigmoid"; state (c, n, m, h) fp32 [B, NH, DH] updated in place
    (zeros when None); status: an optional int32 device tensor that a timed-out wait sets to
    MLSTM_ERR_TIMEOUT.  Returns (h_seq [B, S, NH, DH] or None, (c, n, m, h)).
    """
    if forget not in ("exp", "sigmoid"):
        raise ValueError("forget must be 'exp' or 'sigmoid'")
    lib = load()
    B, S, _, NH, DH = wx.shape
    if state is None:
        state = tuple(torch.zeros((B, NH, DH), dtype=torch.float32, device=wx.device) for _ in range(4))
    c, n, m, h = state
    if want_h and h_out is None:
        h_out = torch.empty((B, S, NH, DH), dtype=wx.dtype, device=wx.device)
    st = lib.slstm_fwd(_ptr(wx), _ptr(R), _dt(wx), B, S, NH, DH, 1 if forget == "sigmoid" else 0, _ptr(c), _ptr(n),
                       _ptr(m), _ptr(h), _ptr(h_out if want_h else None), _ptr(status), _stream(stream))
    _check("slstm_fwd", st)
    return (h_out if want_h else None), (c, n, m, h)


def slstm_batch_per_cluster(B, NH, DH, dtype) -> int:
    dt = MLSTM_BF16 if dtype == torch.bfloat16 else MLSTM_F32
    return int(load().slstm_batch_per_cluster(B, NH, DH, dt))
