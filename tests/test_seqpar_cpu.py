"""Sequence-parallel forward pass on CPU ranks (gloo): the protocol of
xlstm_mlstm_cell_b200.seqpar with the fp64 oracle standing in for the kernels.

Each rank holds one slice of the sequence; the slices' zero-start final states and
log decay sums are all-gathered and composed into each rank's start state.  The
test checks that the slices' h, run from those start states, equal the oracle's
single pass over the whole sequence, and that the last rank's state is the whole
sequence's final state (as exp(m) C, exp(m) n: the stabilizer may differ).
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from xlstm_mlstm_cell_b200 import seqpar
from xlstm_mlstm_cell_b200.workloads import make_custom


def _logsigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def _compose(C_parts, n_parts, m_parts, g_parts, rank):
    """The start state of slice `rank`: slices 0 .. rank-1 composed from the zero state."""
    C = np.zeros(C_parts.shape[1:])
    n = np.zeros(n_parts.shape[1:])
    m = np.zeros(m_parts.shape[1:])
    for r in range(rank):
        g, mr = np.asarray(g_parts[r], np.float64), np.asarray(m_parts[r], np.float64)
        mn = np.maximum(m + g, mr)
        a, b = np.exp(m + g - mn), np.exp(mr - mn)
        C = a[..., None, None] * C + b[..., None, None] * np.asarray(C_parts[r], np.float64)
        n = a[..., None] * n + b[..., None] * np.asarray(n_parts[r], np.float64)
        m = mn
    return C, n, m


class OracleOps:
    """CPU stand-ins for the kernels: the oracle, a logsigmoid sum and the composition."""

    @staticmethod
    def final_state(k, v, igate, fgate, chunk):
        B, NH, S, dk = k.shape
        q = torch.zeros_like(k)
        _, C, n, m = oracle.run(q, k, v, igate, fgate, None, want_h=False, nthreads=1)
        return torch.from_numpy(C).float(), torch.from_numpy(n).float(), torch.from_numpy(m).float()

    @staticmethod
    def log_decay_sum(fgate):
        return torch.from_numpy(_logsigmoid(fgate.numpy()).sum(-1)).float()

    @staticmethod
    def state_prefix(C_parts, n_parts, m_parts, g_parts, rank):
        C, n, m = _compose(C_parts.numpy(), n_parts.numpy(), m_parts.numpy(), g_parts.numpy(), rank)
        return torch.from_numpy(C).float(), torch.from_numpy(n).float(), torch.from_numpy(m).float()

    @staticmethod
    def fwd_state(q, k, v, igate, fgate, ogate, chunk, state):
        C0, n0, m0 = state
        h, C, n, m = oracle.run(q, k, v, igate, fgate, ogate, C=C0.numpy(), n=n0.numpy(), m=m0.numpy(),
                                nthreads=1)
        return torch.from_numpy(h), (torch.from_numpy(C), torch.from_numpy(n), torch.from_numpy(m))


SHAPE = dict(B=1, NH=2, DHQK=8, DHV=8)


def _inputs(S):
    return make_custom(SHAPE["B"], SHAPE["NH"], S, SHAPE["DHQK"], SHAPE["DHV"], "f32", seed=31, ig=(-1.0, 2.0),
                       fg=(2.0, 1.5))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, S, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, i, f, o = _inputs(S)
        L = S // world
        sl = slice(rank * L, (rank + 1) * L)
        cut = lambda x: x[:, :, sl].contiguous()
        h, (C, n, m) = seqpar.fwd_sequence_parallel(cut(q), cut(k), cut(v), cut(i), cut(f), cut(o), chunk=16,
                                                    ops=OracleOps())
        results[rank] = (h.numpy(), C.numpy(), n.numpy(), m.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_protocol_on_cpu_ranks(world):
    S = 12 * world
    with mp.get_context("spawn").Manager() as man:
        results = man.dict()
        mp.spawn(_worker, args=(world, _free_port(), S, results), nprocs=world, join=True)
        res = dict(results)
    q, k, v, i, f, o = _inputs(S)
    hr, Cr, nr, mr = oracle.run(q, k, v, i, f, o, nthreads=1)
    h = np.concatenate([res[r][0] for r in range(world)], axis=2)
    assert np.abs(h - hr).max() <= 1e-5 * np.abs(hr).max()
    _, C, n, m = res[world - 1]
    eC, eCr = np.exp(m)[..., None, None] * C, np.exp(mr)[..., None, None] * Cr
    en, enr = np.exp(m)[..., None] * n, np.exp(mr)[..., None] * nr
    assert np.abs(eC - eCr).max() <= 1e-5 * np.abs(eCr).max()
    assert np.abs(en - enr).max() <= 1e-5 * np.abs(enr).max()


def test_composition_of_slices_equals_one_pass():
    """The identity the state-prefix kernel implements, on the oracle in fp64: composing the
    zero-start final states of consecutive slices gives the state of one pass (as exp(m) C)."""
    S, cuts = 40, [0, 7, 19, 40]
    q, k, v, i, f, o = _inputs(S)
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        cut = lambda x: x[:, :, a:b].contiguous()
        _, C, n, m = oracle.run(cut(q), cut(k), cut(v), cut(i), cut(f), None, want_h=False, nthreads=1)
        parts.append((C, n, m, _logsigmoid(cut(f).numpy()).sum(-1)))
    C_parts, n_parts, m_parts, g_parts = (np.stack([p[j] for p in parts]) for j in range(4))
    C, n, m = _compose(C_parts, n_parts, m_parts, g_parts, len(parts))
    _, Cr, nr, mr = oracle.run(q, k, v, i, f, None, want_h=False, nthreads=1)
    eC, eCr = np.exp(m)[..., None, None] * C, np.exp(mr)[..., None, None] * Cr
    assert np.abs(eC - eCr).max() <= 1e-12 * np.abs(eCr).max()
    assert np.abs(np.exp(m)[..., None] * n - np.exp(mr)[..., None] * nr).max() <= \
        1e-12 * np.abs(np.exp(mr)[..., None] * nr).max()
    assert np.all(m >= mr - 1e-12)      # the composed stabilizer is never below the one-pass one
