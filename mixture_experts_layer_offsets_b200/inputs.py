"""Seeded synthetic inputs for the MoE FFN layer: shapes, distributions, seeds.

This module holds no arithmetic of the method.  It only draws random tensors
in a fixed order from a seeded ``torch.Generator`` so that the CUDA path and the
float64 oracle receive the very same values.

Workloads (T tokens, d_model, E experts, top_k, expert d_ff):

* ``tiny_f32``        T=512,   d=256,  E=8,   k=2, f=512,  fp32; router std d**-0.5
* ``bf16_e8``         T=16384, d=2048, E=8,   k=4, f=1024, bf16; router std 1e-4
* ``bf16_e128``       as ``bf16_e8`` with E=128 (16x the expert parameters)
* ``bf16_skew_e128``  T=32768, d=2048, E=128, k=4, f=1024, bf16; router std
  d**-0.5 plus a per-expert logit bias of std 2 (heavy-tailed counts with empty
  experts); compared against a padded capacity of 1.25x the mean load
* ``mxfp8_e128``      T=32768, d=4096, E=128, k=4, f=1536; bf16 activations,
  fp32 master weights, MXFP8 operands; router std 1e-4

Distributions: x ~ N(0, 1); router weight ~ N(0, router_std**2); expert
weights ~ N(0, 0.02**2); upstream gradient ~ N(0, 1).  Draw order from one
generator seeded with ``seed``: x, w_router, bias, w1, w2, dout.  The
near-uniform router (std 1e-4) gives random routing; the skewed workload uses
std d**-0.5 so that the bias does not decide every token alone.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["MoEConfig", "CONFIGS", "make_inputs", "shrink"]


@dataclass(frozen=True)
class MoEConfig:
    name: str
    dtype: str          # "f32" | "bf16" | "mxfp8"
    T: int
    d_model: int
    E: int
    top_k: int
    d_ff: int
    router_std: float
    bias_std: float = 0.0
    w_std: float = 0.02
    padded_cf: tuple | None = None   # capacity factor as (num, den)

    @property
    def R(self) -> int:
        return self.T * self.top_k

    @property
    def act_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def weight_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


CONFIGS = {
    "tiny_f32": MoEConfig("tiny_f32", "f32", 512, 256, 8, 2, 512, 1.0 / math.sqrt(256)),
    "bf16_e8": MoEConfig("bf16_e8", "bf16", 16384, 2048, 8, 4, 1024, 1e-4),
    "bf16_e128": MoEConfig("bf16_e128", "bf16", 16384, 2048, 128, 4, 1024, 1e-4),
    "bf16_skew_e128": MoEConfig("bf16_skew_e128", "bf16", 32768, 2048, 128, 4, 1024,
                                1.0 / math.sqrt(2048), bias_std=2.0, padded_cf=(5, 4)),
    "mxfp8_e128": MoEConfig("mxfp8_e128", "mxfp8", 32768, 4096, 128, 4, 1536, 1e-4),
}


def shrink(cfg: MoEConfig, **kw) -> MoEConfig:
    """A copy of ``cfg`` with some sizes replaced (for small parity cases)."""
    return replace(cfg, **kw)


def make_inputs(cfg: MoEConfig, device="cpu", seed: int = 0) -> dict:
    """Draw x, w_router, bias, w1 [E, 2f, d], w2 [E, d, f], dout for ``cfg``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    T, d, E, f = cfg.T, cfg.d_model, cfg.E, cfg.d_ff

    def randn(*shape, std=1.0):
        t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        return t.mul_(std) if std != 1.0 else t

    x = randn(T, d)
    w_router = randn(E, d, std=cfg.router_std)
    bias = randn(E, std=cfg.bias_std) if cfg.bias_std else None
    w1 = randn(E, 2 * f, d, std=cfg.w_std)
    w2 = randn(E, d, f, std=cfg.w_std)
    dout = randn(T, d)
    act, wt = cfg.act_dtype, cfg.weight_dtype
    return dict(
        x=x.to(act), w_router=w_router.to(act), bias=bias,
        w1=w1.to(wt), w2=w2.to(wt), dout=dout.to(act),
    )
