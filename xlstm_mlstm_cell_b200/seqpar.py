"""Sequence-parallel mlstm_fwd over a torch.distributed process group.

Rank r of R holds the r-th of R consecutive slices of the sequence (every head, the
same slice length on every rank).  One call runs the three steps declared in
include/mlstm.h:

1. the slice's final state from the zero state (mlstm_fwd_final_state) and its total
   log forget decay (mlstm_log_decay_sum);
2. one all-gather of these summaries over the group (packed into one tensor: one
   collective per call, NCCL over NVLink between GPUs);
3. the slice's start state from the summaries of the slices before it
   (mlstm_state_prefix), then mlstm_fwd_state over the slice from it.

Every step of the arithmetic runs in the library's kernels; this module only moves
tensors and calls the binding.  The operations are injectable (``ops``) so that the
multi-rank logic can be exercised on CPU ranks with stand-ins.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from xlstm_mlstm_cell_b200 import binding


class CudaOps:
    """The library's entry points (device tensors)."""

    @staticmethod
    def final_state(k, v, igate, fgate, chunk):
        return binding.fwd_final_state(k, v, igate, fgate, chunk=chunk)

    @staticmethod
    def log_decay_sum(fgate):
        return binding.log_decay_sum(fgate)

    @staticmethod
    def state_prefix(C_parts, n_parts, m_parts, g_parts, rank):
        return binding.state_prefix(C_parts, n_parts, m_parts, g_parts, rank)

    @staticmethod
    def fwd_state(q, k, v, igate, fgate, ogate, chunk, state):
        h, C, n, m = binding.fwd(q, k, v, igate, fgate, ogate, chunk=chunk, state=state)
        return h, (C, n, m)


def pack_summary(C, n, m, g):
    """One flat float32 tensor holding a slice's summary (C, n, m, g)."""
    return torch.cat([C.reshape(-1), n.reshape(-1), m.reshape(-1), g.reshape(-1)])


def unpack_summaries(flat, R, B, NH, DHQK, DHV):
    """Inverse of pack_summary over R concatenated summaries: (C_parts, n_parts, m_parts, g_parts)."""
    sizes = [B * NH * DHQK * DHV, B * NH * DHQK, B * NH, B * NH]
    per = sum(sizes)
    rows = flat.reshape(R, per)
    C, n, m, g = torch.split(rows, sizes, dim=1)
    return (C.reshape(R, B, NH, DHQK, DHV).contiguous(), n.reshape(R, B, NH, DHQK).contiguous(),
            m.reshape(R, B, NH).contiguous(), g.reshape(R, B, NH).contiguous())


def fwd_sequence_parallel(q, k, v, igate, fgate, ogate=None, chunk: int = 64, group=None, ops=None):
    """This rank's slice of the forward pass over the whole sequence.

    q, k ``[B, NH, S_r, DHQK]``, v, ogate ``[B, NH, S_r, DHV]``, gates ``[B, NH, S_r]``: the
    rank's slice.  Returns ``(h, (C, n, m))``: h for the slice and the state after it (on the
    last rank, the final state of the whole sequence; its stabilizer m can be above that of a
    single pass, with C and n scaled to match).
    """
    ops = ops or CudaOps()
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, NH, _, DHQK = k.shape
    DHV = v.shape[-1]
    C_r, n_r, m_r = ops.final_state(k, v, igate, fgate, chunk)
    g_r = ops.log_decay_sum(fgate)
    mine = pack_summary(C_r, n_r, m_r, g_r)
    parts = [torch.empty_like(mine) for _ in range(R)]
    dist.all_gather(parts, mine, group=group)
    C_parts, n_parts, m_parts, g_parts = unpack_summaries(torch.cat(parts), R, B, NH, DHQK, DHV)
    start = ops.state_prefix(C_parts, n_parts, m_parts, g_parts, rank)
    return ops.fwd_state(q, k, v, igate, fgate, ogate, chunk, start)
