"""mlstm_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Some callers may not call cudaMalloc or any allocating routine (a host framework
that owns all device memory and gives out no scratch, or a latency-critical path
that cannot afford an allocation's implicit synchronization).  mlstm_fwd_noalloc
serves them from a scratch array built into the library.  These tests call it
through the C ABI and check it against mlstm_fwd, with the parity tolerances of
the other tests, on two calls in a row (the second call finds the first call's
data in the shared scratch array).  This file is collected last on purpose.
"""
from __future__ import annotations

import pytest
import torch

from tests.parity import TOL, rel_l2
from xlstm_mlstm_cell_b200 import binding
from xlstm_mlstm_cell_b200.workloads import make_custom


def test_oversize_shape_is_rejected_before_any_launch():
    """A shape needing more scratch than the built-in array returns MLSTM_ERR_WORKSPACE."""
    lib = binding.load()
    B, NH, S, DK, DV, ch = 1, 8, 8192, 256, 512, 64
    need = lib.mlstm_fwd_workspace_size(B, NH, S, DK, DV, ch, binding.MLSTM_BF16)
    assert need > binding.NOALLOC_MAX_BYTES
    fake = 1 << 20   # never dereferenced: the call returns before touching the GPU
    st = lib.mlstm_fwd_noalloc(fake, fake, fake, fake, fake, None, binding.MLSTM_BF16, B, NH, S, DK, DV, ch,
                               fake, None, None, None, None)
    assert st == 3


@pytest.mark.gpu
@pytest.mark.parametrize("B,NH,S,DK,DV,ch,dt", [(1, 4, 1024, 256, 256, 64, "bf16"),
                                                 (1, 2, 700, 256, 512, 128, "bf16"),   # the paired walk
                                                 (1, 2, 100, 32, 32, 16, "f32")])
def test_noalloc_matches_fwd_on_two_calls_in_a_row(cuda_lib, B, NH, S, DK, DV, ch, dt):
    need = binding.workspace_size(B, NH, S, DK, DV, ch, torch.bfloat16 if dt == "bf16" else torch.float32)
    assert 0 < need <= binding.NOALLOC_MAX_BYTES
    for call, seed in enumerate((31, 32)):
        inputs = [None if x is None else x.cuda() for x in
                  make_custom(B, NH, S, DK, DV, dt, seed=seed, ig=(-1.0, 2.0), fg=(4.0, 1.0))]
        ref = binding.fwd(*inputs, chunk=ch)
        out = binding.fwd_noalloc(*inputs, chunk=ch)
        torch.cuda.synchronize()
        for name, x, r in zip("hCnm", out, ref):
            err = rel_l2(x.cpu(), r.cpu())
            assert err <= TOL[dt], "call %d, %s: rel-L2 %.3e" % (call, name, err)


@pytest.mark.gpu
def test_noalloc_status_after_a_completed_call(cuda_lib):
    """mlstm_fwd_noalloc_status reads the status word that the last no-alloc call left in the
    built-in array: MLSTM_OK after a call that ran to completion."""
    inputs = [None if x is None else x.cuda() for x in
              make_custom(1, 2, 300, 128, 128, "bf16", seed=33, ig=(-1.0, 2.0), fg=(4.0, 1.0))]
    binding.fwd_noalloc(*inputs, chunk=64)
    assert binding.fwd_noalloc_status() == 0
    binding.fwd_noalloc(*inputs, chunk=128)
    assert binding.fwd_noalloc_status() == 0
