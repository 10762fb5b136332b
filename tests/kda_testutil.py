"""Helpers for the GPU parity tests: run the oracle on chosen (sequence, head)
pairs of a packed batch and compare with the max|err| / max|ref| metric."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle

TOL_BF16 = 2e-2   # bf16 inputs, fp32 state (the stated parity bar)
TOL_F32 = 1e-4    # fp32-input check mode


def relerr(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    denom = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (denom if denom > 0 else 1.0))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def token_index(cu_host, seqs):
    cu = [int(x) for x in cu_host]
    return torch.cat([torch.arange(cu[n], cu[n + 1]) for n in seqs]) if seqs else torch.zeros(0, dtype=torch.long)


def oracle_subset(inp: dict, seqs, heads, gate: str = "bounded"):
    """Oracle on every token of sequences ``seqs`` for heads ``heads``.

    Returns ``(o [T_sub, len(heads), dv], S [len(seqs), len(heads), dk, dv], tok)``
    where ``tok`` are the packed token indices of the chosen sequences.
    """
    cu = [int(x) for x in inp["cu_seqlens_host"]]
    tok = token_index(cu, seqs)
    hs = torch.tensor(heads, dtype=torch.long)
    dev = inp["q"].device

    def pick(t):
        return t.index_select(0, tok.to(dev)).index_select(1, hs.to(dev)).cpu()

    lens = [cu[n + 1] - cu[n] for n in seqs]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s0 = None
    if inp.get("initial_state") is not None:
        s0 = inp["initial_state"].index_select(0, torch.tensor(seqs, device=dev)) \
                                 .index_select(1, hs.to(dev)).cpu()
    o, S = oracle.prefill(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["z"]),
                          inp["A"].index_select(0, hs.to(dev)).cpu(), pick(inp["beta"]),
                          sub_cu, s0, gate=gate)
    return o, S, tok


def gpu_subset(o_gpu, S_gpu, tok, seqs, heads):
    hs = torch.tensor(heads, dtype=torch.long, device=o_gpu.device)
    o = o_gpu.index_select(0, tok.to(o_gpu.device)).index_select(1, hs)
    S = S_gpu.index_select(0, torch.tensor(seqs, device=S_gpu.device)).index_select(1, hs)
    return to_np(o), to_np(S)
