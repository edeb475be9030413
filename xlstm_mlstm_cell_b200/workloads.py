"""Seeded synthetic workloads for the mLSTM cell (shapes, distributions, seeds).

This module holds no arithmetic of the method: it only draws random tensors.
Both the tests (for the CUDA path and for the oracle) and the benchmark take
their inputs from here.  Every tensor is drawn in float32 on the CPU from a
``torch.Generator`` seeded with the workload's seed, in the order q, k, v,
input gate, forget gate, output gate, and then rounded to bf16 (round to
nearest even) where the workload is bf16.  Gates stay float32.  Layouts are
``[B, NH, S, D]`` and ``[B, NH, S]``.

The five workloads are the ones the library is measured and checked on:

* ``fwd_f32_small``   fp32, B1 NH2 S64 d16/16 chunk 16 (parity only)
* ``fwd_bf16_d256``   bf16, B4 NH4 S2048 d256/256 chunk 64, no output gate
* ``fwd_bf16_7b``     bf16, B1 NH8 S8192 d256/512 chunk 64 (a 7B-shaped prefill)
* ``fwd_bf16_long``   bf16, B1 NH8 S131072 d256/512 chunk 128 (long context)
* ``step_bf16``       decode: B256 NH8 d256/512 fp32 state from a 512-token
                      prefill, then 1000 one-token steps
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "f32" or "bf16": type of q, k, v, o and h
    B: int
    NH: int
    S: int              # tokens of the forward pass (prefill length for the decode workload)
    DHQK: int
    DHV: int
    chunk: int
    qkv_scale: float    # q, k, v ~ qkv_scale * N(0, 1)
    ig: tuple           # input-gate pre-activation ~ N(mean, std)
    fg: tuple           # forget-gate pre-activation ~ N(mean, std)
    ogate: bool         # output gate present: o = sigmoid(N(0, 1))
    seed: int
    steps: int = 0      # decode steps (decode workload only)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "fwd_f32_small": Workload("fwd_f32_small", "f32", 1, 2, 64, 16, 16, 16, 1.0, (0.0, 1.0), (3.0, 1.0), True, 1001),
    "fwd_bf16_d256": Workload("fwd_bf16_d256", "bf16", 4, 4, 2048, 256, 256, 64, 1.0, (0.0, 1.0), (3.0, 1.5), False, 1002),
    "fwd_bf16_7b": Workload("fwd_bf16_7b", "bf16", 1, 8, 8192, 256, 512, 64, 0.5, (-1.0, 2.0), (4.0, 1.0), True, 1003),
    "fwd_bf16_long": Workload("fwd_bf16_long", "bf16", 1, 8, 131072, 256, 512, 128, 0.5, (-1.0, 2.0), (6.0, 1.0), True, 1004),
    # decode: the state comes from a 512-token prefill drawn like fwd_bf16_7b (qkv scale 0.5);
    # the step tokens use q, k, v ~ N(0, 1) and the same gate distributions.
    "step_bf16": Workload("step_bf16", "bf16", 256, 8, 512, 256, 512, 64, 0.5, (-1.0, 2.0), (4.0, 1.0), True, 1005, steps=1000),
}


def draw(shape_qk, shape_v, shape_g, dtype, qkv_scale, ig, fg, ogate, gen):
    """Draws (q, k, v, igate, fgate, ogate) in the fixed order from ``gen``."""
    q = torch.randn(shape_qk, generator=gen) * qkv_scale
    k = torch.randn(shape_qk, generator=gen) * qkv_scale
    v = torch.randn(shape_v, generator=gen) * qkv_scale
    i = torch.randn(shape_g, generator=gen) * ig[1] + ig[0]
    f = torch.randn(shape_g, generator=gen) * fg[1] + fg[0]
    o = torch.sigmoid(torch.randn(shape_v, generator=gen)) if ogate else None
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    if o is not None:
        o = o.to(dtype)
    return q, k, v, i.contiguous(), f.contiguous(), o


def make_fwd_inputs(w: Workload, S: int | None = None, B: int | None = None, NH: int | None = None):
    """Forward-pass inputs of workload ``w`` on the CPU (sizes overridable)."""
    S = w.S if S is None else S
    B = w.B if B is None else B
    NH = w.NH if NH is None else NH
    gen = torch.Generator().manual_seed(w.seed)
    return draw((B, NH, S, w.DHQK), (B, NH, S, w.DHV), (B, NH, S), w.torch_dtype,
                w.qkv_scale, w.ig, w.fg, w.ogate, gen)


def make_step_inputs(w: Workload, step: int, B: int | None = None, NH: int | None = None):
    """Token inputs of decode step ``step`` (q, k, v ~ N(0, 1)), ``[B, NH, D]``."""
    B = w.B if B is None else B
    NH = w.NH if NH is None else NH
    gen = torch.Generator().manual_seed(w.seed * 100003 + 7 + step)
    return draw((B, NH, w.DHQK), (B, NH, w.DHV), (B, NH), w.torch_dtype,
                1.0, w.ig, w.fg, w.ogate, gen)


def make_dh(B, NH, S, DHV, dtype, seed):
    """The gradient of a loss with respect to h, dh ~ N(0, 1) [B, NH, S, DHV], for the backward pass
    (drawn from its own generator, seeded with ``seed``)."""
    gen = torch.Generator().manual_seed(seed)
    dt = torch.float32 if dtype in ("f32", torch.float32) else torch.bfloat16
    return torch.randn((B, NH, S, DHV), generator=gen).to(dt)


def make_custom(B, NH, S, DHQK, DHV, dtype, seed, qkv_scale=1.0, ig=(0.0, 1.0), fg=(3.0, 1.0),
                ogate=True):
    """Free-form inputs for sweeps and edge cases."""
    gen = torch.Generator().manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return draw((B, NH, S, DHQK), (B, NH, S, DHV), (B, NH, S), dt, qkv_scale, ig, fg, ogate, gen)


# ---------------------------------------------------------------- sLSTM recurrence

@dataclasses.dataclass(frozen=True)
class SlstmWorkload:
    """Inputs of the sLSTM recurrence: gate pre-activations wx [B, S, 4, NH, DH] (gate order
    i, f, z, o; i, z, o ~ N(0, 1), f ~ N(f_loc, 1)) and recurrent weights R [NH, 4, DH, DH]
    ~ N(0, 1 / DH), so that R h is of order one."""
    name: str
    dtype: str
    B: int
    S: int
    NH: int
    DH: int
    forget: str         # "exp" or "sigmoid"
    f_loc: float
    seed: int

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# a 4-head sLSTM layer of a 1024-wide model over 1024 tokens, 16 sequences; sigmoid forget gate
# with pre-activations ~ N(3, 1) (forget gates near 0.95, a slowly decaying memory)
SLSTM_WORKLOADS = {
    "slstm_f32": SlstmWorkload("slstm_f32", "f32", 16, 1024, 4, 256, "sigmoid", 3.0, 1006),
}


def make_slstm_inputs(B, S, NH, DH, dtype, seed, f_loc=3.0):
    """(wx, R) on the CPU, drawn in that order from a generator seeded with ``seed``."""
    gen = torch.Generator().manual_seed(seed)
    wx = torch.randn(B, S, 4, NH, DH, generator=gen)
    wx[:, :, 1] += f_loc
    R = torch.randn(NH, 4, DH, DH, generator=gen) / DH ** 0.5
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return wx.to(dt), R.to(dt)
