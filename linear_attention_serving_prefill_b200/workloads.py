"""Seeded synthetic inputs for the KDA mixer.

This module only draws random numbers and shapes them: it holds none of the
mixer's arithmetic, and both the CUDA path and the CPU oracle take their inputs
from here.  The distributions are the ones the pages' configurations state
(post-projection tensors, i.e. what the mixer receives):

* q, k ~ N(0, 1), then scaled to unit L2 norm per (token, head) -- the input
  branch ends in L2Norm ("Kimi K3: Architecture, Training, and Million-Token
  Agentic RL", section 3.2 input equations);
* v ~ N(0, 1); z ~ N(0, 1) per (token, head, key channel);
* beta = sigmoid(N(0, 1)) per (token, head), fp32;
* A ~ U(-1, 1) per (head, key channel), fp32;
* initial states 0, or N(0, 0.02^2) fp32 where a configuration asks for them;
* varlen lengths round(exp(U(ln 1024, ln 65536))).

Draw order for a given seed: lengths, q, k, v, z, beta logits, A, initial state.
q, k, v, z are drawn in fp32 and rounded once (round-to-nearest-even) to the
storage dtype; the rounded tensors are what both sides consume.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

__all__ = ["PrefillConfig", "DecodeConfig", "CONFIGS", "prefill_inputs",
           "decode_inputs", "varlen_lengths", "config_inputs"]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    lengths: tuple            # one entry per packed sequence (may be resolved from a seed)
    H: int
    dk: int
    dv: int
    dtype: str                # "bf16" or "f32": storage dtype of q, k, v, z, o
    s0_std: float = 0.0       # 0 -> no initial state (zeros)
    write_final: bool = True
    seed: int = 0


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    dtype: str
    steps: int
    nsets: int = 16           # step s uses input set s mod nsets
    state_std: float = 0.02
    seed: int = 4


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> List[int]:
    """n lengths, log-uniform in [lo, hi], rounded to integers (seeded)."""
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))))
            for x in u]


CONFIGS = {
    "tiny_f32": PrefillConfig("tiny_f32 (B=1,H=2,T=64,d=32,fp32)", (64,), 2, 32, 32,
                              "f32", seed=0),
    "prefill_4k": PrefillConfig("prefill_4k (B=1,H=32,T=4096,d=128,bf16)", (4096,), 32,
                                128, 128, "bf16", seed=1),
    "prefill_32k": PrefillConfig("prefill_32k (B=1,H=96,T=32768,d=128,bf16)", (32768,),
                                 96, 128, 128, "bf16", seed=2),
    "varlen_resume": PrefillConfig(
        "varlen_resume (16 seqs log-uniform 1K-64K,H=96,d=128,bf16,S0~N(0,0.02^2))",
        tuple(varlen_lengths(16, 1024, 65536, seed=3)), 96, 128, 128, "bf16",
        s0_std=0.02, seed=3),
    "decode_256": DecodeConfig("decode_256 (B=256,H=96,d=128,bf16,1000 steps)", 256, 96,
                               128, 128, "bf16", steps=1000, seed=4),
}


def _dt(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def prefill_inputs(lengths, H: int, dk: int, dv: int, dtype: str = "bf16", seed: int = 0,
                   s0_std: float = 0.0, device="cpu", z_mean: float = 0.0,
                   z_std: float = 1.0, beta_value: Optional[float] = None) -> dict:
    """Packed varlen prefill inputs.

    Returns a dict with q, k, z [T,H,dk] and v [T,H,dv] in the storage dtype,
    beta [T,H] fp32, A [H,dk] fp32, cu_seqlens [N+1] int32 (on ``device``),
    cu_seqlens_host (a CPU copy), and initial_state [N,H,dk,dv] fp32 or None.
    ``z_mean``/``z_std``/``beta_value`` only exist to build edge cases.
    """
    lengths = [int(x) for x in lengths]
    N, T = len(lengths), sum(lengths)
    g = torch.Generator(device=device).manual_seed(seed)
    dt = _dt(dtype)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    q = _unit_rows(torch.randn(T, H, dk, **f32)).to(dt)
    k = _unit_rows(torch.randn(T, H, dk, **f32)).to(dt)
    v = torch.randn(T, H, dv, **f32).to(dt)
    z = (torch.randn(T, H, dk, **f32) * z_std + z_mean).to(dt)
    blog = torch.randn(T, H, **f32)
    beta = torch.sigmoid(blog) if beta_value is None else torch.full_like(blog, beta_value)
    A = torch.rand(H, dk, **f32) * 2.0 - 1.0
    s0 = torch.randn(N, H, dk, dv, **f32) * s0_std if s0_std > 0 else None
    cu = torch.zeros(N + 1, dtype=torch.int32)
    if N:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    return dict(q=q, k=k, v=v, z=z, beta=beta.contiguous(), A=A, cu_seqlens=cu.to(device),
                cu_seqlens_host=cu, initial_state=s0, lengths=lengths)


def config_inputs(cfg: PrefillConfig, device="cpu") -> dict:
    return prefill_inputs(cfg.lengths, cfg.H, cfg.dk, cfg.dv, cfg.dtype, cfg.seed,
                          cfg.s0_std, device)


def decode_inputs(B: int, H: int, dk: int, dv: int, dtype: str = "bf16", seed: int = 4,
                  nsets: int = 16, pool: Optional[int] = None, state_std: float = 0.02,
                  device="cpu", permute_slots: bool = False) -> dict:
    """Decode-step inputs: ``nsets`` per-step sets stacked on a leading axis.

    q, k, z [nsets,B,H,dk], v [nsets,B,H,dv] (storage dtype); beta [nsets,B,H]
    fp32; A [H,dk] fp32; state pool [P,H,dk,dv] fp32 ~ N(0, state_std^2);
    slots [B] int32 (identity, or a seeded permutation into a larger pool).
    """
    P = B if pool is None else pool
    g = torch.Generator(device=device).manual_seed(seed)
    dt = _dt(dtype)
    f32 = dict(dtype=torch.float32, device=device, generator=g)
    q = _unit_rows(torch.randn(nsets, B, H, dk, **f32)).to(dt)
    k = _unit_rows(torch.randn(nsets, B, H, dk, **f32)).to(dt)
    v = torch.randn(nsets, B, H, dv, **f32).to(dt)
    z = torch.randn(nsets, B, H, dk, **f32).to(dt)
    beta = torch.sigmoid(torch.randn(nsets, B, H, **f32))
    A = torch.rand(H, dk, **f32) * 2.0 - 1.0
    state = torch.randn(P, H, dk, dv, **f32) * state_std
    if permute_slots:
        slots = torch.randperm(P, generator=torch.Generator().manual_seed(seed + 1))[:B]
    else:
        slots = torch.arange(B)
    return dict(q=q, k=k, v=v, z=z, beta=beta, A=A, state=state,
                slots=slots.to(torch.int32).to(device))
