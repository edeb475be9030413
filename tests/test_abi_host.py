"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/mlstm.h declares, and rejects bad arguments before touching the GPU."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from xlstm_mlstm_cell_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    names = []
    for fname in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fname.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fname)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b((?:mlstm|slstm)_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "mlstm_fwd" in names and "mlstm_step" in names and "slstm_fwd" in names
    for name in names:
        assert hasattr(lib, name), name
        assert name in binding.SIGNATURES, "binding lacks " + name


def test_status_strings(lib):
    for code in range(6):
        s = lib.mlstm_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.mlstm_status_string(0) == b"ok"


def test_bwd_tensor_path_query(lib):
    """Which backward products run on the tensor cores: bf16, chunk 64 or 128, head sizes % 128."""
    bf, f32 = binding.MLSTM_BF16, binding.MLSTM_F32
    assert lib.mlstm_bwd_tensor_path(256, 512, 64, bf) == 1
    assert lib.mlstm_bwd_tensor_path(128, 128, 128, bf) == 1
    assert lib.mlstm_bwd_tensor_path(256, 512, 32, bf) == 0     # chunk
    assert lib.mlstm_bwd_tensor_path(64, 512, 64, bf) == 0      # DHQK % 128
    assert lib.mlstm_bwd_tensor_path(256, 192, 64, bf) == 0     # DHV % 128
    assert lib.mlstm_bwd_tensor_path(256, 512, 64, f32) == 0    # fp32 inputs stay on the CUDA cores
    assert lib.mlstm_bwd_tensor_path(12, 512, 64, bf) == -1
    assert lib.mlstm_bwd_tensor_path(256, 512, 48, bf) == -1
    # the tensor-core path's workspace keeps the chunk-start states, the scores and g as bf16 parts
    # instead of fp32, the state gradients only as bf16 and adds bf16 copies: 2 DHQK DHV + 2 chunk^2
    # bytes less per chunk and head and 4 DHQK + 4 DHV more per token and head; its walk leaves
    # DHQK DHV / 2048 partial sums of E_c per chunk and head instead of one (here every array is a
    # multiple of 256 bytes)
    B, NH, S, DK, DV, ch = 1, 8, 8192, 256, 512, 64
    extra = lib.mlstm_bwd_workspace_size(B, NH, S, DK, DV, ch, bf) - lib.mlstm_bwd_workspace_size(B, NH, S, DK, DV, ch, f32)
    NC = S // ch
    assert extra == (-B * NH * NC * (2 * DK * DV + 2 * ch * ch) + B * NH * S * (4 * DK + 4 * DV)
                     + B * NH * NC * 4 * (DK * DV // 2048 - 1))


@pytest.mark.parametrize("DK,DV,ch,dt", [(64, 128, 64, "f32"), (96, 40, 32, "f32"), (128, 256, 64, "bf16"),
                                          (256, 512, 128, "bf16")])
def test_bwd_workspace_formula(lib, DK, DV, ch, dt):
    """mlstm_bwd_workspace_size equals the byte counts include/mlstm.h documents: a 256-byte status
    word, 4 bytes per head for the last chunk stabilizer, and per chunk and head and per token and
    head (with 64 heads every array is a multiple of 256 bytes, so no alignment padding enters)."""
    B, NH, S = 1, 64, 1000
    NC, BH = -(-S // ch), B * NH
    ntk, njt = -(-DK // 32), -(-DV // 64)
    code = binding.MLSTM_BF16 if dt == "bf16" else binding.MLSTM_F32
    tc = lib.mlstm_bwd_tensor_path(DK, DV, ch, code) == 1
    assert tc == (dt == "bf16")
    if tc:
        per_chunk = 6 * DK * DV + DK * DV // 512 + 8 * DK + 6 * ch * ch + 12
        per_token = 4 * DK + 8 * DV + 12 * ntk + 4 * njt + 24
    else:
        per_chunk = 8 * DK * (DV + 1) + 8 * ch * ch + 16
        per_token = 4 * DV + 12 * ntk + 4 * njt + 24
    expected = 256 + 4 * BH + BH * NC * per_chunk + BH * S * per_token
    assert lib.mlstm_bwd_workspace_size(B, NH, S, DK, DV, ch, code) == expected


def test_workspace_size(lib):
    ws = lib.mlstm_fwd_workspace_size(1, 8, 8192, 256, 512, 64, binding.MLSTM_BF16)
    assert ws > 0 and ws % 256 == 0
    assert lib.mlstm_fwd_workspace_size(1, 8, 8192, 256, 512, 48, binding.MLSTM_BF16) == 0   # chunk
    assert lib.mlstm_fwd_workspace_size(1, 8, 8192, 12, 512, 64, binding.MLSTM_BF16) == 0    # DHQK % 8
    assert lib.mlstm_fwd_workspace_size(1, 8, 8192, 256, 1024, 64, binding.MLSTM_BF16) == 0  # DHV > 512
    assert lib.mlstm_fwd_workspace_size(-1, 8, 8192, 256, 512, 64, binding.MLSTM_BF16) == 0
    assert lib.mlstm_fwd_workspace_size(1, 8, 8192, 256, 512, 64, 7) == 0                    # dtype
    assert lib.mlstm_fwd_workspace_size(1, 8, 0, 256, 512, 64, binding.MLSTM_BF16) > 0
    # beyond the sizes mlstm_fwd accepts (B * NH > 2^30, which would also overflow an int): 0
    assert lib.mlstm_fwd_workspace_size(1 << 16, 1 << 15, 64, 64, 64, 64, binding.MLSTM_BF16) == 0
    assert lib.mlstm_fwd_workspace_size(1 << 15, 1 << 15, 64, 64, 64, 64, binding.MLSTM_BF16) > 0


FAKE = 1 << 20   # a 16-byte-aligned non-NULL address that is never dereferenced


def fwd_args(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, ig=FAKE, fg=FAKE, og=None, dt=binding.MLSTM_BF16, B=1, NH=2, S=128,
             DHQK=64, DHV=64, chunk=64, h=FAKE, C=None, n=None, m=None, ws=FAKE, wsb=1 << 40, stream=None)
    a.update(over)
    return a


def call_fwd(lib, a):
    return lib.mlstm_fwd(a["q"], a["k"], a["v"], a["ig"], a["fg"], a["og"], a["dt"], a["B"], a["NH"], a["S"],
                         a["DHQK"], a["DHV"], a["chunk"], a["h"], a["C"], a["n"], a["m"], a["ws"], a["wsb"],
                         a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(ig=None), 1), (dict(fg=None), 1),
    (dict(h=None), 1), (dict(q=FAKE + 4), 1), (dict(og=FAKE + 8), 1), (dict(C=FAKE + 2), 1),
    (dict(B=-1), 1), (dict(S=-5), 1), (dict(dt=3), 2), (dict(chunk=48), 2), (dict(chunk=256), 2),
    (dict(DHQK=12), 2), (dict(DHV=520), 2), (dict(DHQK=0), 2),
    (dict(ws=None), 3), (dict(wsb=100), 3), (dict(ws=FAKE + 16), 1),
])
def test_fwd_rejects_bad_arguments(lib, over, expect):
    assert call_fwd(lib, fwd_args(**over)) == expect


def step_args(**over):
    a = dict(C=FAKE, n=FAKE, m=FAKE, q=FAKE, k=FAKE, v=FAKE, ig=FAKE, fg=FAKE, og=None, dt=binding.MLSTM_BF16,
             B=2, NH=2, DHQK=64, DHV=64, h=FAKE, stream=None)
    a.update(over)
    return a


def call_step(lib, a):
    return lib.mlstm_step(a["C"], a["n"], a["m"], a["q"], a["k"], a["v"], a["ig"], a["fg"], a["og"], a["dt"],
                          a["B"], a["NH"], a["DHQK"], a["DHV"], a["h"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(C=None), 1), (dict(n=None), 1), (dict(m=None), 1), (dict(q=None), 1), (dict(h=None), 1),
    (dict(C=FAKE + 4), 1), (dict(og=FAKE + 4), 1), (dict(B=-2), 1), (dict(dt=9), 2),
    (dict(DHQK=10), 2), (dict(DHV=2), 2), (dict(DHV=2048), 2), (dict(DHQK=1024), 2),
])
def test_step_rejects_bad_arguments(lib, over, expect):
    assert call_step(lib, step_args(**over)) == expect


def test_empty_batch_is_a_no_op(lib):
    # B * NH == 0 enqueues nothing for the step and returns before any launch
    assert call_step(lib, step_args(B=0, C=None, n=None, m=None)) == 0


def test_fwd_state_needs_the_whole_state(lib):
    a = fwd_args()
    st = lib.mlstm_fwd_state(a["q"], a["k"], a["v"], a["ig"], a["fg"], a["og"], a["dt"], a["B"], a["NH"], a["S"],
                             a["DHQK"], a["DHV"], a["chunk"], FAKE, None, FAKE, a["h"], None, None, None, a["ws"],
                             a["wsb"], None)
    assert st == 1
    st = lib.mlstm_fwd_state(a["q"], a["k"], a["v"], a["ig"], a["fg"], a["og"], a["dt"], a["B"], a["NH"], a["S"],
                             a["DHQK"], a["DHV"], a["chunk"], FAKE + 4, FAKE, FAKE, a["h"], None, None, None, a["ws"],
                             a["wsb"], None)
    assert st == 1


def test_fwd_status_rejects_null(lib):
    assert lib.mlstm_fwd_status(None, None) == 1


def test_tensor_path_query(lib):
    bf, f32 = binding.MLSTM_BF16, binding.MLSTM_F32
    assert lib.mlstm_fwd_tensor_path(256, 512, 64, bf) == 1
    assert lib.mlstm_fwd_tensor_path(64, 128, 128, bf) == 1
    assert lib.mlstm_fwd_tensor_path(256, 512, 64, f32) == 0     # fp32 inputs: CUDA-core path
    assert lib.mlstm_fwd_tensor_path(256, 200, 64, bf) == 0      # DHV not a multiple of 128
    assert lib.mlstm_fwd_tensor_path(256, 512, 32, bf) == 0      # chunk 32
    assert lib.mlstm_fwd_tensor_path(256, 512, 48, bf) == -1     # unsupported chunk
    assert lib.mlstm_fwd_tensor_path(256, 512, 64, 7) == -1      # unsupported dtype


def test_paired_walk_query(lib):
    bf, f32 = 1, 0
    assert lib.mlstm_fwd_paired_walk(256, 512, 128, bf) == 1     # the long-context shape
    assert lib.mlstm_fwd_paired_walk(256, 256, 128, bf) == 1
    assert lib.mlstm_fwd_paired_walk(256, 384, 128, bf) == 0     # DHV not a multiple of 256
    assert lib.mlstm_fwd_paired_walk(256, 512, 64, bf) == 0      # chunk 64: one CTA per value tile
    assert lib.mlstm_fwd_paired_walk(128, 512, 128, bf) == 0     # DHQK 128
    assert lib.mlstm_fwd_paired_walk(256, 512, 128, f32) == -1   # fp32: CUDA-core path
    assert lib.mlstm_fwd_paired_walk(256, 512, 48, bf) == -1     # unsupported chunk


def test_kernel_launch_counts(lib):
    bf, f32 = binding.MLSTM_BF16, binding.MLSTM_F32
    # gate preprocessing is one kernel up to 4096 tokens per head, two beyond
    assert lib.mlstm_fwd_kernel_launches(4, 4, 2048, 256, 256, 64, bf) == 1 + 3
    assert lib.mlstm_fwd_kernel_launches(4, 4, 4096, 256, 256, 64, bf) == 1 + 3
    assert lib.mlstm_fwd_kernel_launches(1, 8, 4097, 256, 512, 64, bf) == 2 + 3
    assert lib.mlstm_fwd_kernel_launches(1, 8, 131072, 256, 512, 128, bf) == 2 + 3
    assert lib.mlstm_fwd_kernel_launches(1, 2, 64, 16, 16, 16, f32) == 1 + 2
    assert lib.mlstm_fwd_kernel_launches(1, 2, 64 * 200, 16, 16, 64, f32) == 2 + 2
    assert lib.mlstm_fwd_kernel_launches(0, 2, 64, 16, 16, 16, f32) == 0


def slstm_args(**over):
    a = dict(wx=FAKE, R=FAKE, dt=0, B=2, S=5, NH=2, DH=64, fs=0, c=FAKE, n=FAKE, m=FAKE, h=FAKE, ho=FAKE, st=None)
    a.update(over)
    return a


def call_slstm(lib, a):
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return lib.slstm_fwd(v(a["wx"]), v(a["R"]), a["dt"], a["B"], a["S"], a["NH"], a["DH"], a["fs"], v(a["c"]),
                         v(a["n"]), v(a["m"]), v(a["h"]), v(a["ho"]), v(a["st"]), None)


@pytest.mark.parametrize("over,expect", [
    (dict(wx=None), 1), (dict(R=None), 1), (dict(c=None), 1), (dict(n=None), 1), (dict(m=None), 1),
    (dict(h=None), 1), (dict(R=FAKE + 8), 1), (dict(wx=FAKE + 2), 1), (dict(dt=1, wx=FAKE + 1), 1),
    (dict(c=FAKE + 2), 1), (dict(B=-1), 1), (dict(S=-3), 1), (dict(NH=0), 1), (dict(dt=7), 2),
    (dict(DH=48), 2), (dict(DH=512), 2), (dict(DH=16), 2), (dict(st=FAKE + 2), 1),
])
def test_slstm_rejects_bad_arguments(lib, over, expect):
    assert call_slstm(lib, slstm_args(**over)) == expect


def test_slstm_empty_work_is_a_no_op(lib):
    # nothing to run: no launch, and the pointers are not looked at
    assert call_slstm(lib, slstm_args(B=0, wx=None, R=None, c=None, n=None, m=None, h=None, ho=None)) == 0
    assert call_slstm(lib, slstm_args(S=0, wx=None, R=None, ho=None)) == 0


def test_slstm_batch_per_cluster_rejects_unsupported(lib):
    assert lib.slstm_batch_per_cluster(4, 2, 48, 0) == 0
    assert lib.slstm_batch_per_cluster(4, 0, 64, 0) == 0
    assert lib.slstm_batch_per_cluster(4, 2, 64, 5) == 0


# ---------------------------------------------------------------- launch failures (no GPU)
# On a machine without a CUDA device every launch fails.  Calls with valid arguments must then
# return MLSTM_ERR_CUDA (4) through the launch-error path instead of crashing; the fake device
# pointers are never dereferenced on the host.  Skipped where a device is present, since there
# the fake pointers would reach real kernels.
def _no_device():
    import torch
    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_device(), reason="needs a machine without a CUDA device")
@pytest.mark.parametrize("over", [
    dict(),                                        # tensor-core path (bf16, d 64, chunk 64)
    dict(dt=binding.MLSTM_F32, chunk=16),          # fp32 CUDA-core path
    dict(S=5000, DHQK=128, DHV=128, chunk=128),    # gate preprocessing in two kernels
])
def test_fwd_reports_launch_failure(lib, over):
    assert call_fwd(lib, fwd_args(**over)) == 4


@pytest.mark.skipif(not _no_device(), reason="needs a machine without a CUDA device")
def test_step_and_slstm_report_launch_failure(lib):
    assert call_step(lib, step_args()) == 4
    assert call_slstm(lib, slstm_args()) == 4
    assert lib.slstm_batch_per_cluster(4, 2, 64, 0) == 0      # no device to size the clusters for


# ---------------------------------------------------------------- sequence-parallel pieces, profiled fwd
def test_log_decay_sum_rejects_bad_arguments(lib):
    v = ctypes.c_void_p
    assert lib.mlstm_log_decay_sum(v(FAKE), -1, 2, 8, v(FAKE), None) == 1
    assert lib.mlstm_log_decay_sum(v(FAKE), 1, 2, -8, v(FAKE), None) == 1
    assert lib.mlstm_log_decay_sum(v(FAKE), 1, 2, 8, None, None) == 1          # no output
    assert lib.mlstm_log_decay_sum(None, 1, 2, 8, v(FAKE), None) == 1          # tokens but no gates
    assert lib.mlstm_log_decay_sum(None, 0, 2, 8, None, None) == 0             # no heads: no launch


def _prefix(lib, **over):
    a = dict(Cp=FAKE, np_=FAKE, mp=FAKE, gp=FAKE, R=2, rank=1, B=1, NH=2, DK=64, DV=64, C0=FAKE, n0=FAKE, m0=FAKE)
    a.update(over)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return lib.mlstm_state_prefix(v(a["Cp"]), v(a["np_"]), v(a["mp"]), v(a["gp"]), a["R"], a["rank"], a["B"],
                                  a["NH"], a["DK"], a["DV"], v(a["C0"]), v(a["n0"]), v(a["m0"]), None)


@pytest.mark.parametrize("over,expect", [
    (dict(R=0), 1), (dict(rank=2), 1), (dict(rank=-1), 1), (dict(B=-1), 1),
    (dict(DK=12), 2), (dict(DV=1024), 2), (dict(C0=None), 1), (dict(m0=None), 1),
    (dict(Cp=None), 1), (dict(gp=None), 1), (dict(C0=FAKE + 4), 1), (dict(Cp=FAKE + 8), 1),
])
def test_state_prefix_rejects_bad_arguments(lib, over, expect):
    assert _prefix(lib, **over) == expect


def test_state_prefix_empty_batch_is_a_no_op(lib):
    assert _prefix(lib, B=0, C0=None, n0=None, m0=None) == 0


def test_final_state_checks_only_the_inputs_it_reads(lib):
    v = ctypes.c_void_p
    args = lambda k, vv, i, f, ws, wsb: lib.mlstm_fwd_final_state(k, vv, i, f, binding.MLSTM_BF16, 1, 2, 128, 64, 64,
                                                                     64, None, None, None, ws, wsb, None)
    assert args(None, v(FAKE), v(FAKE), v(FAKE), v(FAKE), 1 << 40) == 1        # k missing
    assert args(v(FAKE + 4), v(FAKE), v(FAKE), v(FAKE), v(FAKE), 1 << 40) == 1 # k misaligned
    assert args(v(FAKE), v(FAKE), v(FAKE), v(FAKE), None, 1 << 40) == 3        # no workspace


def test_profiled_needs_the_event_array(lib):
    a = fwd_args()
    st = lib.mlstm_fwd_profiled(a["q"], a["k"], a["v"], a["ig"], a["fg"], a["og"], a["dt"], a["B"], a["NH"], a["S"],
                                a["DHQK"], a["DHV"], a["chunk"], a["h"], a["C"], a["n"], a["m"], a["ws"], a["wsb"],
                                a["stream"], None)
    assert st == 1


# ---------------------------------------------------------------- concurrent host callers (no GPU)
@pytest.mark.skipif(not _no_device(), reason="needs a machine without a CUDA device")
def test_concurrent_host_callers(lib):
    """Eight host threads call the library at once (ctypes releases the GIL): the host-side caches
    (per-kernel shared-memory limits, the tensor-map encoder, the sLSTM cluster capacity, the
    no-alloc array's address) are filled under a lock, and every call returns its status."""
    import threading
    results, errors = [], []

    def worker(tid):
        try:
            for it in range(20):
                ws = lib.mlstm_fwd_workspace_size(1, 8, 4096 + tid, 256, 512, 64, binding.MLSTM_BF16)
                assert ws > 0 and ws % 256 == 0
                r = [call_fwd(lib, fwd_args()),
                     call_fwd(lib, fwd_args(dt=binding.MLSTM_F32, chunk=16)),
                     call_fwd(lib, fwd_args(DHQK=256, DHV=512, chunk=128)),
                     call_step(lib, step_args()),
                     call_slstm(lib, slstm_args(DH=32 << (it % 4))),
                     lib.mlstm_fwd_noalloc_status(None)]
                results.append(tuple(r))
        except Exception as e:   # noqa: BLE001 - reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert len(results) == 8 * 20
    assert set(results) == {(4, 4, 4, 4, 4, 4)}


@pytest.mark.skipif(not _no_device(), reason="needs a machine without a CUDA device")
def test_noalloc_status_without_device(lib):
    assert lib.mlstm_fwd_noalloc_status(None) == 4
