"""Seeded synthetic inputs for the SSD scan and decode step.

This module draws random numbers and nothing else: it holds none of the
scan's arithmetic, so both the CUDA path's tests and the fp64 oracle can take
their inputs from it.

Workloads (shapes of the nnterp guide "Mamba-2" example for the 130m layer --
heads 24, head_dim 64, state_dim 128, groups 1, chunk 256 -- up to larger
layers and long context):

  c0_tiny_fp32   b=1  L=64     H=4  P=16 N=16  G=1 Q=16   fp32 inputs
  c1_130m        b=4  L=2048   H=24 P=64 N=128 G=1 Q=256  bf16 x/B/C
  c2_2p7b        b=8  L=4096   H=80 P=64 N=128 G=1 Q=256  bf16, D ~ N(1, 0.1)
  c3_long        b=1  L=65536  H=80 P=64 N=128 G=8 Q=256  bf16, init state N(0, 0.1)
  c4_decode      b=256 H=80 P=64 N=128 G=8, 512 decode steps, state N(0, 0.1)

Distributions: x, B, C ~ N(0, 1); dt_raw ~ N(0, 1) (fp32);
dt_bias[h] = softplus^-1(v), v log-uniform on [1e-3, 0.1] (the dt_bias
initialisation of the "Mamba-2 dt_bias initialization bug" page, Method
section); A[h] = -exp(u), u uniform on [ln 1, ln 16]; D = 1 unless stated.
"N(m, s)" is read with s the standard deviation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class ScanConfig:
    name: str
    batch: int
    seqlen: int
    nheads: int
    head_dim: int
    state_dim: int
    ngroups: int
    chunk_size: int
    dtype: str = "bf16"          # storage dtype of x, B, C: "f32" or "bf16"
    d_dist: str = "ones"         # "ones" or "normal" (N(1, 0.1))
    init: str = "zero"           # "zero" (no initial state) or "normal" (N(0, 0.1))
    seed: int = 0

    def with_(self, **kw) -> "ScanConfig":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclass(frozen=True)
class StepConfig:
    name: str
    batch: int
    nheads: int
    head_dim: int
    state_dim: int
    ngroups: int
    steps: int
    dtype: str = "bf16"
    d_dist: str = "ones"
    seed: int = 4

    def with_(self, **kw) -> "StepConfig":
        return replace(self, **kw)


SCAN_CONFIGS: Dict[str, ScanConfig] = {
    "c0_tiny_fp32": ScanConfig("c0_tiny_fp32", 1, 64, 4, 16, 16, 1, 16, "f32", "ones", "zero", 0),
    "c1_130m": ScanConfig("c1_130m", 4, 2048, 24, 64, 128, 1, 256, "bf16", "ones", "zero", 1),
    "c2_2p7b": ScanConfig("c2_2p7b", 8, 4096, 80, 64, 128, 1, 256, "bf16", "normal", "zero", 2),
    "c3_long": ScanConfig("c3_long", 1, 65536, 80, 64, 128, 8, 256, "bf16", "ones", "normal", 3),
}

STEP_CONFIGS: Dict[str, StepConfig] = {
    "c4_decode": StepConfig("c4_decode", 256, 80, 64, 128, 8, 512, "bf16", "ones", 4),
}

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}
_SEED_OFFSET = 0x55D0


def storage_dtype(name: str) -> torch.dtype:
    return _DT[name]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_SEED_OFFSET + int(seed))
    return g


def _head_params(g: torch.Generator, H: int, d_dist: str):
    # dt_bias = softplus^-1(v), v = exp(U(ln 1e-3, ln 0.1)); softplus^-1(v) = v + log(-expm1(-v))
    u = torch.rand(H, generator=g, dtype=torch.float64)
    v = torch.exp(math.log(1e-3) + u * (math.log(0.1) - math.log(1e-3)))
    dt_bias = (v + torch.log(-torch.expm1(-v))).float()
    ua = torch.rand(H, generator=g, dtype=torch.float64)
    A = (-torch.exp(ua * math.log(16.0))).float()
    if d_dist == "ones":
        D = torch.ones(H, dtype=torch.float32)
    elif d_dist == "normal":
        D = 1.0 + 0.1 * torch.randn(H, generator=g, dtype=torch.float32)
    else:
        raise ValueError(d_dist)
    return dt_bias, A, D


def make_scan_inputs(cfg: ScanConfig, seed: Optional[int] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Host (CPU) tensors for one scan call.  x/B/C are in the storage dtype
    (already rounded); dt_raw, dt_bias, A, D, init_state are fp32."""
    g = _gen(cfg.seed if seed is None else seed)
    b, L, H, P, N, G = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    dt_bias, A, D = _head_params(g, H, cfg.d_dist)
    sd = _DT[cfg.dtype]
    x = torch.randn(b, L, H, P, generator=g, dtype=torch.float32).to(sd)
    B = torch.randn(b, L, G, N, generator=g, dtype=torch.float32).to(sd)
    C = torch.randn(b, L, G, N, generator=g, dtype=torch.float32).to(sd)
    dt_raw = torch.randn(b, L, H, generator=g, dtype=torch.float32)
    init = None
    if cfg.init == "normal":
        init = 0.1 * torch.randn(b, H, N, P, generator=g, dtype=torch.float32)
    elif cfg.init != "zero":
        raise ValueError(cfg.init)
    return dict(x=x, dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, init_state=init)


def make_step_inputs(cfg: StepConfig, steps: Optional[int] = None,
                     seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Host tensors for ``steps`` decode tokens: x [T,b,H,P], dt_raw [T,b,H],
    B/C [T,b,G,N] (storage dtype), the initial state [b,H,N,P] fp32 ~ N(0,0.1)
    and the per-head parameters."""
    T = cfg.steps if steps is None else int(steps)
    g = _gen(cfg.seed if seed is None else seed)
    b, H, P, N, G = cfg.batch, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    dt_bias, A, D = _head_params(g, H, cfg.d_dist)
    sd = _DT[cfg.dtype]
    state = 0.1 * torch.randn(b, H, N, P, generator=g, dtype=torch.float32)
    x = torch.randn(T, b, H, P, generator=g, dtype=torch.float32).to(sd)
    B = torch.randn(T, b, G, N, generator=g, dtype=torch.float32).to(sd)
    C = torch.randn(T, b, G, N, generator=g, dtype=torch.float32).to(sd)
    dt_raw = torch.randn(T, b, H, generator=g, dtype=torch.float32)
    return dict(x=x, dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, state=state)


def make_grad_inputs(cfg: ScanConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Host fp32 upstream gradients for a backward call: dy [b,L,H,P] and
    dfinal [b,H,N,P], both N(0, 1)."""
    g = _gen((cfg.seed if seed is None else seed) + 7919)
    b, L, H, P, N = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim
    dy = torch.randn(b, L, H, P, generator=g, dtype=torch.float32)
    dfinal = torch.randn(b, H, N, P, generator=g, dtype=torch.float32)
    return dict(dy=dy, dfinal=dfinal)
