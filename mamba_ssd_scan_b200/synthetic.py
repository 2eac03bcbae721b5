"""Seeded synthetic inputs for the SSD scan workloads.

This module only draws random numbers; it holds none of the scan's arithmetic.
Both the CUDA path's tests/benchmark and the oracle are fed from it.

Distributions (the pages' workloads are HFT-style tick sequences of 256-1024
steps with d_state 64/128 and chunk 256; the proprietary market data they
train on is not available, so these draws stand in for it):

  x, B, C  ~ N(0, 1)
  dt_raw   ~ N(0, 1)
  dt_bias  = softplus^-1(v), v ~ U[1e-3, 0.1]      (inverse-softplus init of
             the dt bias, "MAMBA-2 Implementation Gaps", Gap 3)
  A_h      = -u, u ~ U[1, 16]    (a negative scalar per head)
  D_h      ~ N(0, 1)
  init     ~ N(0, 0.1^2) where a workload carries an initial state

Draw order is fixed: x, dt_raw, B, C, dt_bias, A, D, init.  Everything is drawn
in fp32 on a CPU torch.Generator and then cast to the workload dtype, so the
oracle can read the exact rounded values.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class FwdConfig:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: torch.dtype
    init_state: bool = False
    return_final: bool = False

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    steps: int
    dtype: torch.dtype


FWD_CONFIGS = {
    "fwd_f32_small": FwdConfig("fwd_f32_small", 1, 256, 4, 16, 16, 1, 64, torch.float32),
    "fwd_bf16_b4_L1024": FwdConfig("fwd_bf16_b4_L1024", 4, 1024, 24, 64, 64, 1, 256,
                                   torch.bfloat16),
    "fwd_bf16_b8_L4096_init": FwdConfig("fwd_bf16_b8_L4096_init", 8, 4096, 32, 64, 128, 1,
                                        256, torch.bfloat16, init_state=True,
                                        return_final=True),
    "fwd_bf16_b1_L65536_G8": FwdConfig("fwd_bf16_b1_L65536_G8", 1, 65536, 80, 64, 128, 8,
                                       256, torch.bfloat16),
}
DECODE_CONFIGS = {
    "decode_b256_H80": DecodeConfig("decode_b256_H80", 256, 80, 64, 128, 8, 1024,
                                    torch.bfloat16),
}
@dataclasses.dataclass(frozen=True)
class ConvConfig:
    """The causal depthwise convolution over the concatenated x, B and C
    channels of a Mamba-2 block: channels = nheads*headdim + 2*ngroups*dstate."""
    name: str
    batch: int
    seqlen: int       # 1 for the decode step
    channels: int
    width: int
    dtype: torch.dtype
    steps: int = 0    # decode steps replayed (decode only)
    layers: int = 1   # distinct carried states cycled through (decode only)


CONV_CONFIGS = {
    # the x, B, C channels of the b8 L4096 forward workload (32*64 + 2*128)
    "conv1d_bf16_b8_L4096_C2304": ConvConfig("conv1d_bf16_b8_L4096_C2304", 8, 4096, 2304, 4,
                                             torch.bfloat16),
    # the decode workload's channels (80*64 + 2*8*128); 8 layers' states (176 MB) > L2
    "conv1d_update_b256_C7168": ConvConfig("conv1d_update_b256_C7168", 256, 1, 7168, 4,
                                           torch.bfloat16, steps=1024, layers=8),
}


@dataclasses.dataclass(frozen=True)
class SelConfig:
    """The diagonal-A selective scan: channels = d_inner of the model."""
    name: str
    batch: int
    seqlen: int
    channels: int
    dstate: int
    chunk: int
    dtype: torch.dtype
    steps: int = 0    # decode steps replayed (decode only)
    layers: int = 1   # distinct carried states cycled through (decode only)


SEL_CONFIGS = {
    # the headline model's d_inner (d_model 768, expand 2) with Mamba-1's dstate 16
    "sel_bf16_b4_L1024_D1536_N16": SelConfig("sel_bf16_b4_L1024_D1536_N16", 4, 1024, 1536, 16,
                                             32, torch.bfloat16),
    "sel_update_b256_D1536_N16": SelConfig("sel_update_b256_D1536_N16", 256, 1, 1536, 16, 1,
                                           torch.bfloat16, steps=1024, layers=8),
}
# the seed offset of each workload (seed = 1234 + offset)
SEED_OFFSET = {"fwd_f32_small": 0, "fwd_bf16_b4_L1024": 1, "fwd_bf16_b8_L4096_init": 2,
               "fwd_bf16_b1_L65536_G8": 3, "decode_b256_H80": 4,
               "conv1d_bf16_b8_L4096_C2304": 5, "conv1d_update_b256_C7168": 6,
               "sel_bf16_b4_L1024_D1536_N16": 7, "sel_update_b256_D1536_N16": 8}


def _uniform(gen, shape, lo, hi):
    return torch.rand(shape, generator=gen, dtype=torch.float32) * (hi - lo) + lo


def _inv_softplus(v: torch.Tensor) -> torch.Tensor:
    v64 = v.double()
    return (v64 + torch.log(-torch.expm1(-v64))).float()


def head_params(gen: torch.Generator, nheads: int):
    """dt_bias, A, D per head (fp32), drawn in the fixed order."""
    dt_bias = _inv_softplus(_uniform(gen, (nheads,), 1e-3, 0.1))
    A = -_uniform(gen, (nheads,), 1.0, 16.0)
    D = torch.randn((nheads,), generator=gen, dtype=torch.float32)
    return dt_bias, A, D


def make_fwd_inputs(batch, seqlen, nheads, headdim, dstate, ngroups, dtype,
                    seed: int, init_state: bool = False) -> dict:
    """CPU tensors for one forward call (x, dt, B, C in ``dtype``; A, D,
    dt_bias, init_state fp32)."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn((batch, seqlen, nheads, headdim), generator=gen).to(dtype)
    dt = torch.randn((batch, seqlen, nheads), generator=gen).to(dtype)
    B = torch.randn((batch, seqlen, ngroups, dstate), generator=gen).to(dtype)
    C = torch.randn((batch, seqlen, ngroups, dstate), generator=gen).to(dtype)
    dt_bias, A, D = head_params(gen, nheads)
    init = None
    if init_state:
        init = torch.randn((batch, nheads, headdim, dstate), generator=gen) * 0.1
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D, dt_bias=dt_bias, init_state=init)


def make_config_inputs(cfg: FwdConfig, seed: int | None = None) -> dict:
    if seed is None:
        seed = 1234 + SEED_OFFSET.get(cfg.name, 0)
    return make_fwd_inputs(cfg.batch, cfg.seqlen, cfg.nheads, cfg.headdim, cfg.dstate,
                           cfg.ngroups, cfg.dtype, seed, cfg.init_state)


def make_decode_params(batch, nheads, headdim, dstate, seed: int) -> dict:
    """Initial fp32 state ~ N(0, 0.1^2) and the per-head parameters."""
    gen = torch.Generator().manual_seed(seed)
    dt_bias, A, D = head_params(gen, nheads)
    state = torch.randn((batch, nheads, headdim, dstate), generator=gen) * 0.1
    return dict(state=state, A=A, D=D, dt_bias=dt_bias)


def make_decode_step(batch, nheads, headdim, dstate, ngroups, dtype, seed: int,
                     step: int) -> dict:
    """Inputs of one decode step (x, dt, B, C in ``dtype``)."""
    gen = torch.Generator().manual_seed(seed * 1_000_003 + step)
    x = torch.randn((batch, nheads, headdim), generator=gen).to(dtype)
    dt = torch.randn((batch, nheads), generator=gen).to(dtype)
    B = torch.randn((batch, ngroups, dstate), generator=gen).to(dtype)
    C = torch.randn((batch, ngroups, dstate), generator=gen).to(dtype)
    return dict(x=x, dt=dt, B=B, C=C)


def make_gate(shape, dtype, seed: int) -> torch.Tensor:
    """The optional output gate z ~ N(0, 1), of x's shape (drawn from its own
    generator, so the other inputs of a seed are unchanged)."""
    gen = torch.Generator().manual_seed(seed + 7919)
    return torch.randn(tuple(shape), generator=gen, dtype=torch.float32).to(dtype)


def make_norm_inputs(rows: int, channels: int, dtype, seed: int, gate: bool = True) -> dict:
    """Inputs of the gated RMSNorm: y, z ~ N(0, 1) [rows, channels] in dtype
    (z None without the gate) and the weight ~ 1 + 0.1 N(0, 1) [channels]
    fp32 (an RMSNorm weight starts at one)."""
    gen = torch.Generator().manual_seed(seed + 7927)
    y = torch.randn((rows, channels), generator=gen).to(dtype)
    z = torch.randn((rows, channels), generator=gen).to(dtype) if gate else None
    weight = 1.0 + 0.1 * torch.randn((channels,), generator=gen)
    return {"y": y, "z": z, "weight": weight}


def make_bwd_grads(x_shape, state_shape, dtype, seed: int) -> dict:
    """Incoming gradients of a backward call: dy ~ N(0,1) shaped like x (in
    dtype) and d_final ~ N(0,1) shaped like the state (fp32)."""
    gen = torch.Generator().manual_seed(seed + 7907)
    dy = torch.randn(x_shape, generator=gen).to(dtype)
    d_final = torch.randn(state_shape, generator=gen)
    return dict(dy=dy, d_final=d_final)


def make_selective_inputs(batch, seqlen, channels, dstate, dtype, seed: int,
                          init_state: bool = False) -> dict:
    """Inputs of the diagonal-A selective scan: x, dt_raw, B, C ~ N(0,1) in
    dtype; A[d,n] = -exp(A_log) with A_log = log(n+1) + U[-0.5, 0.5] (the
    log(1..N) initialisation, perturbed per channel); dt_bias =
    softplus^-1(U[1e-3, 0.1]); D ~ N(0,1); init ~ N(0, 0.1^2) (fp32)."""
    gen = torch.Generator().manual_seed(seed + 65537)
    x = torch.randn((batch, seqlen, channels), generator=gen).to(dtype)
    dt = torch.randn((batch, seqlen, channels), generator=gen).to(dtype)
    B = torch.randn((batch, seqlen, dstate), generator=gen).to(dtype)
    C = torch.randn((batch, seqlen, dstate), generator=gen).to(dtype)
    a_log = torch.log(torch.arange(1, dstate + 1, dtype=torch.float32)).expand(channels, dstate)
    A = -torch.exp(a_log + _uniform(gen, (channels, dstate), -0.5, 0.5))
    dt_bias = _inv_softplus(_uniform(gen, (channels,), 1e-3, 0.1))
    D = torch.randn((channels,), generator=gen)
    init = torch.randn((batch, channels, dstate), generator=gen) * 0.1 if init_state else None
    return dict(x=x, dt=dt, A=A.contiguous(), B=B, C=C, D=D, dt_bias=dt_bias, init_state=init)


def make_conv_inputs(batch, seqlen, channels, width, dtype, seed: int,
                     init_state: bool = True) -> dict:
    """Inputs of the causal depthwise convolution: x ~ N(0, 1) [b, L, C] in
    dtype, weight ~ N(0, 1/width) [C, width], bias ~ N(0, 0.1^2) [C] and the
    carried inputs init ~ N(0, 1) [b, C, width-1] (fp32), drawn in that order."""
    gen = torch.Generator().manual_seed(seed + 104729)
    x = torch.randn((batch, seqlen, channels), generator=gen).to(dtype)
    w = torch.randn((channels, width), generator=gen) / width ** 0.5
    bias = torch.randn((channels,), generator=gen) * 0.1
    init = (torch.randn((batch, channels, max(width - 1, 0)), generator=gen)
            if init_state and width > 1 else None)
    return dict(x=x, weight=w, bias=bias, init_state=init)


def nchunks(seqlen: int, chunk: int) -> int:
    return int(math.ceil(seqlen / chunk))
