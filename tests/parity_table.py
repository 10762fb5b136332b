"""Measured parity of every prefill path against the fp64 oracle, as a table.

python -m tests.parity_table [--quick]

For each workload and algorithm, prints max|err| / max|ref| of o and of the
final state over EVERY (token, head) of the workload (the oracle runs once per
workload, in groups of heads, and each GPU path is compared with the same
reference).  The slow-decay rows use z ~ N(-4, 1) and N(-8, 1), where the
state keeps information over thousands of chunks.  The decode row runs the
1000 in-place steps of the 256 x 96 batch and compares 64 sampled
(sequence, head) pairs after the last step.  Test infrastructure: it calls the
oracle, so it lives beside the tests.  Needs a B200.
"""
from __future__ import annotations

import argparse
import json
import sys

import numpy as np
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import (CONFIGS, config_inputs, decode_inputs,
                                                             prefill_inputs)
from oracle import oracle
from tests.kda_testutil import oracle_subset

ALGOS = ("cuda_core", "tensor_core", "tensor_core_split", "auto")


def _supported(algo, x):
    dt, dk, dv = x["q"].dtype, x["q"].shape[2], x["v"].shape[2]
    return not (algo.startswith("tensor_core") and (dt != torch.bfloat16 or dk != 128 or dv != 128))


def prefill_rows(name, x, head_group=8):
    x = {key: (val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val)
         for key, val in x.items()}
    n, H = len(x["lengths"]), x["q"].shape[1]
    outs = {}
    for algo in ALGOS:
        if not _supported(algo, x):
            continue
        o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                             x["cu_seqlens_host"], initial_state=x["initial_state"], algo=algo)
        torch.cuda.synchronize()
        assert K.kda_device_status() == 0
        outs[algo] = (o, S)
    acc = {algo: [0.0, 0.0] for algo in outs}   # max|err| of o and S
    ref_max = [0.0, 0.0]
    seqs = list(range(n))
    for h0 in range(0, H, head_group):
        heads = list(range(h0, min(H, h0 + head_group)))
        ref_o, ref_S, tok = oracle_subset(x, seqs, heads)
        ref_max[0] = max(ref_max[0], float(np.abs(ref_o).max()) if ref_o.size else 0.0)
        ref_max[1] = max(ref_max[1], float(np.abs(ref_S).max()))
        hs = torch.tensor(heads, device="cuda")
        for algo, (o, S) in outs.items():
            go = o.index_select(0, tok.cuda()).index_select(1, hs).double().cpu().numpy()
            gS = S.index_select(1, hs).double().cpu().numpy()
            if go.size:
                acc[algo][0] = max(acc[algo][0], float(np.abs(go - ref_o).max()))
            acc[algo][1] = max(acc[algo][1], float(np.abs(gS - ref_S).max()))
    rows = []
    for algo, (eo, es) in acc.items():
        seg = K.kda_prefill_segments(x["q"].shape[0], n, H, x["q"].shape[2], x["v"].shape[2],
                                     x["q"].dtype, algo)
        rows.append({"workload": name, "algo": algo, "segments": seg,
                     "o": eo / max(ref_max[0], 1e-30), "S": es / max(ref_max[1], 1e-30)})
    return rows


def decode_row(steps=1000):
    """The 1000 in-place decode steps of the 256 x 96 batch (step s uses input
    set s mod 16); an 8 x 8 grid of (sequence, head) pairs replayed by the
    oracle, compared after the last step."""
    cfg = CONFIGS["decode_256"]
    d = decode_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.dtype, seed=cfg.seed, nsets=cfg.nsets,
                      device="cuda")
    bsel, hsel = np.arange(0, 256, 32) + 7, np.arange(0, 96, 12) + 5

    def np64(t):
        return t.detach().to("cpu", torch.float64).numpy()

    ref_state = np64(d["state"])[bsel][:, hsel]
    subsets = [{key: np64(d[key][i])[bsel][:, hsel] for key in ("q", "k", "v", "z", "beta")}
               for i in range(cfg.nsets)]
    A_sub = np64(d["A"])[hsel]
    for s in range(steps):
        i = s % cfg.nsets
        o = K.kda_decode_step(d["q"][i], d["k"][i], d["v"][i], d["z"][i], d["A"], d["beta"][i],
                              d["state"])
        sub = subsets[i]
        ref_o, ref_state = oracle.decode_step(sub["q"], sub["k"], sub["v"], sub["z"], A_sub,
                                              sub["beta"], ref_state)
    torch.cuda.synchronize()
    got_o, got_S = np64(o)[bsel][:, hsel], np64(d["state"])[bsel][:, hsel]
    err = lambda g, r: float(np.abs(g - r).max() / np.abs(r).max())  # noqa: E731
    return [{"workload": "decode_256, 1000 steps, 64 sampled pairs", "algo": "decode_step",
             "segments": 0, "o": err(got_o, ref_o), "S": err(got_S, ref_state)}]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--quick", action="store_true", help="skip the 193K-token varlen workload")
    args = ap.parse_args()
    rows = []
    rows += prefill_rows("tiny_f32", config_inputs(CONFIGS["tiny_f32"]))
    rows += prefill_rows("prefill_4k", config_inputs(CONFIGS["prefill_4k"]))
    rows += prefill_rows("prefill_32k", config_inputs(CONFIGS["prefill_32k"]), head_group=16)
    if not args.quick:
        rows += prefill_rows("varlen_resume", config_inputs(CONFIGS["varlen_resume"]), head_group=4)
    for zm in (-4.0, -8.0):
        rows += prefill_rows(f"slow decay z~N({zm:g},1), 16K x 3 heads, S0 != 0",
                             prefill_inputs([16384], 3, 128, 128, "bf16", seed=40 + int(-zm),
                                            s0_std=0.02, z_mean=zm))
    rows += decode_row()
    rows += prefill_rows("slow decay z~N(-4,1), varlen_resume lengths x 2 heads, S0 != 0",
                         prefill_inputs(CONFIGS["varlen_resume"].lengths, 2, 128, 128, "bf16",
                                        seed=43, s0_std=0.02, z_mean=-4.0))
    print("| workload | path | segments | o | final state |")
    print("|---|---|---:|---:|---:|")
    for r in rows:
        print(f"| {r['workload']} | {r['algo']} | {r['segments']} | {r['o']:.2e} | {r['S']:.2e} |")
    json.dump(rows, sys.stderr)


if __name__ == "__main__":
    main()
