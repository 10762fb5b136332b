"""Head sharding of one packed prefill problem across ranks (host-side slicing).

Heads are independent in the KDA recurrence ("Kimi K3: Architecture, Training,
and Million-Token Agentic RL", section 3.1: one state per head), so a problem
can be split across GPUs by heads with no exchange at all.  The library's entry
points take contiguous ``[T, H, d]`` tensors, so a rank cannot be handed a
strided view of its heads: this module copies each rank's heads into
contiguous tensors of the same layout, and puts the per-rank results back.
It does no arithmetic of the mixer.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch

_PER_HEAD = ("q", "k", "v", "z", "beta")   # [T, H, ...]


def head_shard(world: int, rank: int, H: int) -> List[int]:
    """Heads of rank ``rank``: a contiguous block, the first H % world ranks one larger."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return list(range(lo, lo + base + (1 if rank < extra else 0)))


def shard_inputs(x: Dict[str, Optional[torch.Tensor]], heads: List[int]) -> Dict[str, object]:
    """Contiguous copies of the inputs of ``heads``: q, k, v, z [T, h, d],
    beta [T, h], A [h, dk], initial_state [N, h, dk, dv] or None.  cu_seqlens
    (device and host) are shared by every shard unchanged."""
    if not heads or heads != list(range(heads[0], heads[0] + len(heads))):
        raise ValueError("a shard is a non-empty contiguous block of heads")
    out: Dict[str, object] = {}
    for key in _PER_HEAD:
        t = x[key]
        out[key] = t[:, heads[0]:heads[-1] + 1].contiguous()
    out["A"] = x["A"][heads[0]:heads[-1] + 1].contiguous()
    s0 = x.get("initial_state")
    out["initial_state"] = None if s0 is None else s0[:, heads[0]:heads[-1] + 1].contiguous()
    for key in ("cu_seqlens", "cu_seqlens_host", "lengths"):
        if key in x:
            out[key] = x[key]
    return out


def gather_heads(parts: List[torch.Tensor], dim: int = 1) -> torch.Tensor:
    """Concatenate per-rank results (o [T, h, dv] or states [N, h, dk, dv]) in
    rank order along the head axis."""
    return torch.cat(parts, dim=dim)
