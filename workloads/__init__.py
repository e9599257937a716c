"""Seeded synthetic inputs for the selective scan, shared by the tests, the bench and
the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
scan's arithmetic.  Everything is generated on the CPU with a seeded
``torch.Generator`` in fp32 and then rounded once (round-to-nearest-even) to the
I/O dtype, so the CUDA path and the fp64 oracle see bit-identical inputs.

Recipe (per workload):
  u, z           ~ N(0, 1)                 shape (batch, dim, L)
  B, C           ~ N(0, 1)                 shape (batch, dstate, L)
  delta (raw)    ~ 0.1 * N(0, 1)           shape (batch, dim, L)
  A[d, n]        = -(n + 1)                fp32, shape (dim, dstate)
  D[d]           = 1                       fp32
  delta_bias[d]  = inverse softplus of dt, dt log-uniform in [dt_min, dt_max]
                   (computed in fp64, stored fp32)
  softplus on.
The causal-conv prologue draws weight ~ N(0, 1)/sqrt(width), bias ~ 0.1 N(0, 1) and a
carried-in conv state ~ N(0, 1), fp32.
Scans that continue from a given state (initial_state) draw it ~ N(0, 1), fp32,
shape (batch, dim, dstate), from their own seed.
Decode workloads additionally draw an initial state ~ N(0, 1) of shape
(batch, dim, dstate) in fp32 and a pool of POOL per-step input sets.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

POOL = 8  # decode: step i uses input set i % POOL


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    dstate: int
    seqlen: int          # L for a forward scan; 1 for decode
    io: str              # "f32" or "bf16": dtype of u, delta, z, B, C, y
    dt_min: float
    dt_max: float
    decode_steps: int = 0  # >0: single-token decode chained this many times
    seed: int = 1000

    @property
    def elements(self) -> int:
        """B*D*L for a scan; B*D per step for decode."""
        return self.batch * self.dim * (self.seqlen if self.decode_steps == 0 else 1)


# The five synthetic configurations (Mamba-130M and Mamba-2.8B layer shapes).
WORKLOADS = [
    Workload("tiny_f32_b1_d64_L256", 1, 64, 16, 256, "f32", 1e-3, 1e-1, seed=1000),
    Workload("mamba130m_b8_d1536_L2048", 8, 1536, 16, 2048, "bf16", 1e-3, 1e-1, seed=1001),
    Workload("mamba2p8b_b4_d5120_L2048", 4, 5120, 16, 2048, "bf16", 1e-3, 1e-1, seed=1002),
    Workload("long_b1_d5120_L32768", 1, 5120, 16, 32768, "bf16", 1e-4, 1e-2, seed=1003),
    Workload("decode_b256_d5120", 256, 5120, 16, 1, "bf16", 1e-3, 1e-1, decode_steps=1000, seed=1004),
]
HEADLINE = 2  # the Mamba-2.8B-shaped layer scan


def io_torch_dtype(io: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[io]


def _randn(gen, shape, scale=1.0):
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * scale


def _bias_from_dt(gen, dim, dt_min, dt_max):
    """delta_bias = log(expm1(dt)) with dt log-uniform: the inverse of softplus, so that
    softplus(bias) = dt.  Input recipe only; computed in fp64, stored fp32."""
    r = torch.rand(dim, generator=gen, dtype=torch.float64).numpy()
    dt = np.exp(math.log(dt_min) + r * (math.log(dt_max) - math.log(dt_min)))
    return torch.from_numpy(np.log(np.expm1(dt))).to(torch.float32)


def initial_state(batch, dim, dstate=16, seed=0, scale=1.0):
    """Seeded fp32 initial state (batch, dim, dstate) ~ scale * N(0, 1), for scans that
    continue from a given state."""
    g = torch.Generator().manual_seed(seed)
    return _randn(g, (batch, dim, dstate), scale).contiguous()


def conv_inputs(batch, dim, width=4, seed=0, with_bias=True, with_state=False):
    """Seeded causal-conv parameters: weight (dim, width) ~ N(0, 1) / sqrt(width), bias (dim)
    ~ 0.1 N(0, 1), and optionally a carried-in state (batch, dim, width-1) ~ N(0, 1), all fp32."""
    g = torch.Generator().manual_seed(seed)
    w = _randn(g, (dim, width), 1.0 / math.sqrt(width)).contiguous()
    b = _randn(g, (dim,), 0.1) if with_bias else None
    st = _randn(g, (batch, dim, width - 1)).contiguous() if with_state else None
    return dict(conv_weight=w, conv_bias=b, conv_state_in=st)


def scan_inputs(batch, dim, seqlen, dstate=16, io="bf16", dt_min=1e-3, dt_max=1e-1, seed=0,
                with_z=True, with_D=True, with_bias=True, delta_scale=0.1):
    """Seeded forward-scan inputs (CPU tensors): u, delta, z in the I/O dtype,
    B, C in the I/O dtype, A, D, delta_bias in fp32."""
    g = torch.Generator().manual_seed(seed)
    dt_ = io_torch_dtype(io)
    u = _randn(g, (batch, dim, seqlen)).to(dt_)
    z = _randn(g, (batch, dim, seqlen)).to(dt_)
    B = _randn(g, (batch, dstate, seqlen)).to(dt_)
    C = _randn(g, (batch, dstate, seqlen)).to(dt_)
    delta = _randn(g, (batch, dim, seqlen), delta_scale).to(dt_)
    bias = _bias_from_dt(g, dim, dt_min, dt_max)
    A = -torch.arange(1, dstate + 1, dtype=torch.float32).repeat(dim, 1).contiguous()
    D = torch.ones(dim, dtype=torch.float32)
    return dict(u=u, delta=delta, A=A, B=B, C=C,
                D=D if with_D else None, z=z if with_z else None,
                delta_bias=bias if with_bias else None)


def workload_inputs(w: Workload):
    """Inputs of a forward-scan workload."""
    assert w.decode_steps == 0
    return scan_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.io, w.dt_min, w.dt_max, seed=w.seed)


def decode_inputs(batch, dim, dstate=16, io="bf16", dt_min=1e-3, dt_max=1e-1, seed=0, pool=POOL):
    """Decode inputs: initial fp32 state ~ N(0,1) (batch, dim, dstate) and a pool of
    per-step sets {u, delta, z: (batch, dim); B, C: (batch, dstate)}."""
    g = torch.Generator().manual_seed(seed)
    dt_ = io_torch_dtype(io)
    state0 = _randn(g, (batch, dim, dstate))
    sets = []
    for _ in range(pool):
        sets.append(dict(
            u=_randn(g, (batch, dim)).to(dt_),
            z=_randn(g, (batch, dim)).to(dt_),
            B=_randn(g, (batch, dstate)).to(dt_),
            C=_randn(g, (batch, dstate)).to(dt_),
            delta=_randn(g, (batch, dim), 0.1).to(dt_),
        ))
    bias = _bias_from_dt(g, dim, dt_min, dt_max)
    A = -torch.arange(1, dstate + 1, dtype=torch.float32).repeat(dim, 1).contiguous()
    D = torch.ones(dim, dtype=torch.float32)
    return dict(state0=state0, sets=sets, A=A, D=D, delta_bias=bias)


def workload_decode_inputs(w: Workload):
    assert w.decode_steps > 0
    return decode_inputs(w.batch, w.dim, w.dstate, w.io, w.dt_min, w.dt_max, seed=w.seed)
