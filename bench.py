"""Benchmark of the KDA mixer on B200: chunked prefill (headline) and decode step.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one kda_prefill call over the 32K-token, 96-head workload
(B=1, H=96, T=32768, dk=dv=128, bf16 q/k/v/z, fp32 A/beta/state), inputs
resident in HBM.  Each rank runs its own independent problem (weak scaling, no
collective on the data path).  Rank 0 prints one JSON line with tokens/s,
TFLOP/s, the dominant kernel's roofline, the decode-step GB/s (B=256 cached
states, H=96, in place), an end-to-end figure through the C ABI with pinned
host buffers (steps pipelined over two device slots and three streams), SM
clocks sampled during the timed region, and the CPU oracle timed on a bounded
sample of the same workload.  Legs on the 4K x 32-head workload add the
sequence split and the unbounded-gate cost.

--impl reference times the CPU oracle itself as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KDA prefill tokens/s + TFLOP/s (H=96,d=128,T=32K); decode-step GB/s vs HBM peak"
BYTES_PER_TOKEN_HEAD = 1284        # q,k,v,z bf16 (4*256) + beta fp32 (4) + o bf16 (256)
L2_BYTES = 126 * 1000 * 1000       # B200 L2 (126 MB)
FLOPS_PER_TOKEN_HEAD = 108544      # 6*dk*dv + 16*(3*dk + 2*dv) at dk = dv = 128
FALLBACK_HBM_GBS = 6650.0
# Kernels per prefill call -> (names, algorithmic bytes per token-head of each,
# source file).  Tensor-core path: the intra kernel reads q, k, v, z (bf16) and
# beta and writes a 74,496-byte block per (64-token chunk, head), i.e. 1,164 B
# per token-head; the state kernel reads that block and writes o (bf16).
BLOCK_BYTES_PER_TOKEN_HEAD = 74496 // 64
KERNELS = {
    1: (["prefill_cuda_core_kernel"], [BYTES_PER_TOKEN_HEAD], "kda_prefill_cuda_core.cu"),
    3: (["plan_kernel", "intra_kernel", "state_kernel"],
        [0, 1028 + BLOCK_BYTES_PER_TOKEN_HEAD, BLOCK_BYTES_PER_TOKEN_HEAD + 256],
        "kda_prefill_tc.cu"),
}
FALLBACK_BF16_TFLOPS = 1590.0


def split_kernels(G: int):
    """Kernels of a call split into G segments per sequence, with their
    algorithmic bytes per token-head when a fraction f = (G - 1) / G of the
    chunks lies in segments >= 1: the state kernel reads the blocks of those
    chunks twice (local and transition chains) and writes an E image (256 B/th)
    for them besides o; the correction reads E and reads and writes o there.
    The segment composition moves O(N H G) states, nothing per token."""
    f = (G - 1) / G
    return (["plan_kernel", "intra_kernel", "state_kernel", "compose_kernel", "correct_kernel"],
            [0, 1028 + BLOCK_BYTES_PER_TOKEN_HEAD, BLOCK_BYTES_PER_TOKEN_HEAD * (1 + f) + 256 + 256 * f, 0,
             768 * f], "kda_prefill_tc.cu")


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region."""
    QUERY = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.bus = None
        try:
            p = torch.cuda.get_device_properties(device)
            self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def start(self):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        mine = [r for r in rows if len(r) >= 10 and self.bus
                and r[1].strip().upper().endswith(self.bus[-12:].upper())]
        if not mine and len({r[0] for r in rows if len(r) >= 10}) == 1:
            mine = [r for r in rows if len(r) >= 10]
        if not mine:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[2]) for r in mine if r[2].strip().replace(".", "").isdigit()]
        mx = [float(r[3]) for r in mine if r[3].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in mine for i in range(4)
                          if r[6 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(mine)}


def _code_sha(text: str) -> str:
    """sha256 prefix of C/CUDA source text with its comments, trailing blanks and
    blank lines removed, so that an edit of comments alone keeps the same key."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def _source_sha(name: str) -> str:
    """The `_code_sha` key of one kernel source file of the package."""
    path = os.path.join(ROOT, "linear_attention_serving_prefill_b200", "csrc", name)
    with open(path) as f:
        return _code_sha(f.read())


def _traffic(kernel_file: str, kernel: str, units: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not isinstance(rec, dict) or rec.get("source_sha") != _source_sha(kernel_file):
        return None
    return rec["dram_bytes_per_token_head"] * units


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s independent problem (weak scaling: one problem per GPU)."""
    return base + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's time; every rank takes part (same collective order)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(inp, target_s: float, max_heads: int = 96):
    """Times the fp64 CPU oracle on a bounded sample of the prefill workload:
    the first L tokens of the first h heads, L chosen from a short calibration
    so the timed run takes about target_s seconds.  Returns a dict."""
    from oracle import oracle
    cores = oracle.max_threads()
    h = min(max_heads, inp["q"].shape[1])

    def sample(L):
        sl = slice(0, L)
        args = [inp[key][sl, :h].cpu() for key in ("q", "k", "v", "z")]
        return args + [inp["A"][:h].cpu(), inp["beta"][sl, :h].cpu(),
                       torch.tensor([0, L], dtype=torch.int32)]

    cal = sample(128)
    t0 = time.perf_counter()
    oracle.prefill(*cal)
    rate = h * 128 / (time.perf_counter() - t0)          # token-heads / s
    L = int(max(128, min(inp["q"].shape[0], rate * target_s / h)))
    args = sample(L)
    t0 = time.perf_counter()
    oracle.prefill(*args)
    dt = time.perf_counter() - t0
    th_per_s = h * L / dt
    return {"token_heads_per_s": th_per_s, "tokens_per_s": th_per_s / inp["q"].shape[1],
            "cores": min(h, cores), "seconds": dt,
            "sample": f"first {L} tokens x {h} heads of the 32K workload ({h * L} token-heads, "
                      f"fp64 token-by-token oracle, OpenMP over heads); tokens/s = "
                      f"token-heads/s / 96 heads"}


def run_reference(args):
    """Reference arm: the CPU oracle, timed as it stands on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from linear_attention_serving_prefill_b200.workloads import CONFIGS, config_inputs
    cfg = CONFIGS["prefill_32k"]
    # Inputs: the same distributions; generate only the rows the sample touches.
    from linear_attention_serving_prefill_b200.workloads import prefill_inputs
    per_step = max(2.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    inp = prefill_inputs([2048], cfg.H, cfg.dk, cfg.dv, cfg.dtype, seed=cfg.seed)
    res = None
    for _ in range(args.warmup):
        cpu_oracle_sample(inp, per_step)
    vals = []
    for _ in range(args.steps):
        res = cpu_oracle_sample(inp, per_step)
        vals.append(res["tokens_per_s"])
    value = statistics.median(vals) if vals else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * res["seconds"] if res else None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "global_batch": 1, "seq_len": 32768,
                   "parallelism": "host cores (OpenMP over heads)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": res["cores"] if res else 0,
                         "kind": "oracle", "sample": res["sample"] if res else ""},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def split_leg(K, rank_seed, rank, world, dev, stream, args, max_over_ranks, barrier):
    """The single-sequence 4,096-token, 32-head prefill (32 state chains for 148
    SMs), whole and split into segments by the affine scan.  L2 is flushed
    (a 256 MiB write) before every timed call; each call is timed alone."""
    from dataclasses import replace

    from linear_attention_serving_prefill_b200.workloads import CONFIGS, config_inputs
    cfg = CONFIGS["prefill_4k"]
    x = config_inputs(replace(cfg, seed=rank_seed(cfg.seed, rank)), device=dev)
    T, H = x["q"].shape[0], cfg.H
    o = torch.empty(T, H, cfg.dv, dtype=torch.bfloat16, device=dev)
    S = torch.empty(1, H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {"workload": cfg.name, "tokens": T, "heads": H, "l2": "flushed before every call"}
    reps = 30
    for algo in ("tensor_core", "auto"):
        G = K.kda_prefill_segments(T, 1, H, cfg.dk, cfg.dv, torch.bfloat16, algo)
        nk = K.kda_prefill_kernel_count(T, 1, H, cfg.dk, cfg.dv, torch.bfloat16, algo)
        names = KERNELS[nk][0] if nk != 5 else split_kernels(G)[0]
        ws = torch.empty(max(K.kda_prefill_workspace_size(T, 1, H, cfg.dk, cfg.dv, torch.bfloat16,
                                                          algo), 1), dtype=torch.uint8, device=dev)

        def call(ev=None):
            K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                          x["cu_seqlens_host"], None, final_state=S, o=o, workspace=ws, algo=algo,
                          stream=stream, stage_events=ev)

        for _ in range(args.warmup):
            call()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(reps)]
        for row in evs:
            for e in row:
                e.record(stream)   # creates the CUDA event
        torch.cuda.synchronize()
        barrier()
        for i in range(reps):
            flush.fill_(i & 0xFF)
            call(evs[i])
        torch.cuda.synchronize()
        per = [statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(reps))
               for j in range(nk)]
        ms = max_over_ranks(sum(per), world, dev)
        out["split" if G > 1 else "whole"] = {
            "algo": algo, "segments": G, "ms": ms, "tokens_per_s": T / (ms / 1e3),
            "kernels_ms": dict(zip(names, per))}
        del ws
    if "split" in out and "whole" in out:
        out["speedup"] = out["whole"]["ms"] / out["split"]["ms"]
    del x, o, S, flush
    return out


def gate_leg(K, rank_seed, rank, world, dev, stream, args, max_over_ranks, barrier):
    """The cost the lower bound removes, on the 4,096-token, 32-head prefill:
    the tensor-core path with the K3 gate (dense diagonal 16-token tiles) and
    with the unbounded Softplus gate (off-diagonal sub-tile pairs on tcgen05,
    the diagonal 16 x 16 tiles pair by pair, one exponent per pair and key
    channel, by a separate kernel); and the same two gates on the fp32 CUDA-core
    path.  L2 is flushed before every call."""
    from dataclasses import replace

    from linear_attention_serving_prefill_b200.workloads import CONFIGS, config_inputs
    cfg = CONFIGS["prefill_4k"]
    x = config_inputs(replace(cfg, seed=rank_seed(cfg.seed, rank)), device=dev)
    T, H = x["q"].shape[0], cfg.H
    o = torch.empty(T, H, cfg.dv, dtype=torch.bfloat16, device=dev)
    S = torch.empty(1, H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ws = torch.empty(max(K.kda_prefill_gated_workspace_size(T, 1, H, cfg.dk, cfg.dv, torch.bfloat16,
                                                            "tensor_core", "softplus"), 1),
                     dtype=torch.uint8, device=dev)
    out = {"workload": cfg.name, "l2": "flushed before every call"}
    reps = 5
    for name, algo, gate in (("tensor_core_bounded", "tensor_core", "bounded"),
                             ("tensor_core_softplus", "tensor_core", "softplus"),
                             ("cuda_core_bounded", "cuda_core", "bounded"),
                             ("cuda_core_softplus", "cuda_core", "softplus")):
        def call():
            K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                          x["cu_seqlens_host"], None, final_state=S, o=o, workspace=ws, algo=algo,
                          stream=stream, gate=gate)

        for _ in range(2):
            call()
        torch.cuda.synchronize()
        barrier()
        ts = []
        for i in range(reps):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = max_over_ranks(statistics.median(ts), world, dev)
        out[name] = {"ms": ms, "tokens_per_s": T / (ms / 1e3)}
    # Like for like: the tensor-core path with the diagonal tiles pair by pair
    # (the design before the bound) over the same path with dense diagonal tiles.
    out["diagonal_pair_cost_tensor_core"] = (out["tensor_core_softplus"]["ms"] /
                                             out["tensor_core_bounded"]["ms"])
    out["pair_path_cost_cuda_core"] = out["cuda_core_softplus"]["ms"] / out["cuda_core_bounded"]["ms"]
    del x, o, S, flush, ws
    return out


def decode_leg(K, rank, world, dev, stream, args, hbm_peak, barrier, batch=None):
    """Decode step on B cached states (default the 256 x 96 workload), H=96,
    updated in place: GB/s of state traffic over args.decode_steps steps, then
    speculative verify / replay of 4 drafts on the same batch."""
    from linear_attention_serving_prefill_b200.workloads import CONFIGS, decode_inputs
    from dataclasses import replace
    dcfg = CONFIGS["decode_256"]
    if batch:
        dcfg = replace(dcfg, B=batch, name=dcfg.name.replace("B=256", f"B={batch}"))
    d = decode_inputs(dcfg.B, dcfg.H, dcfg.dk, dcfg.dv, dcfg.dtype, seed=rank_seed(dcfg.seed, rank),
                      nsets=dcfg.nsets, device=dev)
    od = torch.empty(dcfg.B, dcfg.H, dcfg.dv, dtype=torch.bfloat16, device=dev)

    def dstep(i):
        j = i % dcfg.nsets
        K.kda_decode_step(d["q"][j], d["k"][j], d["v"][j], d["z"][j], d["A"], d["beta"][j],
                          d["state"], None, o=od, stream=stream)

    for i in range(args.warmup):
        dstep(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.decode_steps):
        dstep(i)
    e1.record(stream)
    torch.cuda.synchronize()
    dms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.decode_steps
    state_bytes = 2 * dcfg.B * dcfg.H * dcfg.dk * dcfg.dv * 4
    dgbs = state_bytes / (dms / 1e3) / 1e9
    decode = {"config": dcfg.name, "ms_per_step": dms, "state_gbs": dgbs,
              "frac_of_hbm": dgbs / hbm_peak, "steps": args.decode_steps,
              "state_bytes_per_step": state_bytes, "gpu_launches": args.decode_steps}

    # Speculative decoding on the same batch: verify 4 drafts per sequence (state
    # read once, not written), then replay the accepted ones (here all 4).
    Tq = 4
    sq, sk, sv, sz = (d[key][:Tq].permute(1, 0, 2, 3).contiguous() for key in ("q", "k", "v", "z"))
    sbeta = d["beta"][:Tq].permute(1, 0, 2).contiguous()
    so = torch.empty(dcfg.B, Tq, dcfg.H, dcfg.dv, dtype=torch.bfloat16, device=dev)
    for _ in range(args.warmup):
        K.kda_decode_multi(sq, sk, sv, sz, d["A"], sbeta, d["state"], o=so, stream=stream)
    torch.cuda.synchronize()
    barrier()
    reps = 50
    e0.record(stream)
    for _ in range(reps):
        K.kda_decode_multi(sq, sk, sv, sz, d["A"], sbeta, d["state"], o=so, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    vms = max_over_ranks(e0.elapsed_time(e1), world, dev) / reps
    e0.record(stream)
    for _ in range(reps):
        K.kda_decode_multi(sq, sk, sv, sz, d["A"], sbeta, d["state"], update_state=True,
                           want_outputs=False, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    rms = max_over_ranks(e0.elapsed_time(e1), world, dev) / reps
    decode["spec_verify"] = {"drafts": Tq, "ms": vms,
                             "state_read_gbs": state_bytes / 2 / (vms / 1e3) / 1e9,
                             "tokens_per_s": dcfg.B * Tq / (vms / 1e3)}
    decode["spec_replay"] = {"accepted": Tq, "ms": rms,
                             "state_gbs": state_bytes / (rms / 1e3) / 1e9}
    del d, od, so
    return decode


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--algo", default="auto",
                    choices=["auto", "cuda_core", "tensor_core", "tensor_core_split"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="prefill_32k", choices=["prefill_32k", "prefill_4k", "varlen_resume"],
                    help="prefill_4k is the small case used for profiler captures")
    ap.add_argument("--prefill-only", action="store_true",
                    help="skip the decode, end-to-end and CPU legs (profiler captures)")
    ap.add_argument("--decode-only", action="store_true",
                    help="run the decode and speculative legs alone (profiler captures)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="sequences of the decode legs (default: the 256-sequence workload)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.workload == "varlen_resume" and (not args.prefill_only or args.impl == "reference"):
        ap.error("the varlen_resume workload runs the prefill leg alone (--prefill-only)")
    if args.impl == "reference":
        run_reference(args)
        return

    import torch.distributed as dist
    from datetime import timedelta

    from linear_attention_serving_prefill_b200 import binding as K
    from linear_attention_serving_prefill_b200.workloads import (CONFIGS, config_inputs,
                                                                 decode_inputs)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    if args.decode_only:
        hbm_peak = _peaks()[0]
        decode = decode_leg(K, rank, world, dev, torch.cuda.current_stream(), args, hbm_peak,
                            barrier, batch=args.decode_batch or None)
        if rank == 0:
            print(json.dumps({"decode": decode, "gpu": torch.cuda.get_device_name(dev)}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    cfg = CONFIGS[args.workload]
    from dataclasses import replace
    inp = config_inputs(replace(cfg, seed=rank_seed(cfg.seed, rank)), device=dev)
    T, H, dk, dv = inp["q"].shape[0], cfg.H, cfg.dk, cfg.dv
    N = inp["cu_seqlens_host"].numel() - 1
    S0 = inp.get("initial_state")       # resumed sequences start from a cached state
    stream = torch.cuda.current_stream()
    o = torch.empty(T, H, dv, dtype=torch.bfloat16, device=dev)
    S = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    ws_bytes = K.kda_prefill_workspace_size(T, N, H, dk, dv, torch.bfloat16, args.algo)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    nk = K.kda_prefill_kernel_count(T, N, H, dk, dv, torch.bfloat16, args.algo)
    n_seg = K.kda_prefill_segments(T, N, H, dk, dv, torch.bfloat16, args.algo)
    kernel_names, kernel_bytes_per_th, kernel_file = (KERNELS[nk] if nk != 5 else
                                                      split_kernels(n_seg))

    def step(events=None):
        K.kda_prefill(inp["q"], inp["k"], inp["v"], inp["z"], inp["A"], inp["beta"],
                      inp["cu_seqlens"], inp["cu_seqlens_host"], S0, final_state=S, o=o,
                      workspace=ws, algo=args.algo, stream=stream, stage_events=events)

    for _ in range(args.warmup):
        step()
    # One event per kernel boundary per timed step (created by a first record).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    torch.cuda.synchronize()
    total_ms = evs[0][0].elapsed_time(evs[-1][-1])
    per_kernel_ms = [statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                     for j in range(nk)]
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    tokens = T * world
    value = tokens / (ms_per_step / 1e3)
    th = T * H
    tflops = th * FLOPS_PER_TOKEN_HEAD * world / (ms_per_step / 1e3) / 1e12

    hbm_peak, tc_peak, peak_src = _peaks()
    dom = max(range(nk), key=lambda j: per_kernel_ms[j])
    launch_ms = per_kernel_ms[dom]
    # The method's algorithmic bytes (1,284 per token-head: q, k, v, z, beta in,
    # o out) over the dominant kernel's launch time.  The bytes that kernel
    # moves by this design (its own reads plus the intermediate block it
    # writes) are reported beside it under "own_bytes_*", not in "frac".
    # With initial states the 64 KiB state of every (sequence, head) is read and
    # the final one written: 2 x 64 KiB more per (sequence, head).
    state_bytes = 2 * N * H * dk * dv * 4 if S0 is not None else 0
    alg_bytes = th * BYTES_PER_TOKEN_HEAD + state_bytes
    achieved = alg_bytes / (launch_ms / 1e3) / 1e9
    own_bytes = th * kernel_bytes_per_th[dom]
    own_gbs = own_bytes / (launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak,
                "traffic": _traffic(kernel_file, kernel_names[dom], th),
                "kernel": kernel_names[dom], "peak_source": peak_src,
                "algorithmic_bytes_per_launch": alg_bytes,
                "algorithmic_bytes_per_token_head": BYTES_PER_TOKEN_HEAD,
                "own_bytes_per_token_head": kernel_bytes_per_th[dom],
                "own_bytes_gbs": own_gbs, "own_bytes_frac": own_gbs / hbm_peak,
                "kernels_ms": dict(zip(kernel_names, per_kernel_ms))}
    path_gbs = alg_bytes / (ms_per_step / 1e3) / 1e9
    path = {"bytes_per_token_head": BYTES_PER_TOKEN_HEAD, "state_bytes": state_bytes,
            "achieved_gbs": path_gbs,
            "hbm_frac": path_gbs / hbm_peak, "tensor_tflops": tflops / world,
            "tensor_frac": tflops / world / tc_peak, "tensor_peak": tc_peak,
            "roofline_ms": alg_bytes / hbm_peak / 1e6}
    launches = args.steps * nk

    decode = e2e = cpu = ckpt = split = gate_cost = None
    if not args.prefill_only:
        split = split_leg(K, rank_seed, rank, world, dev, stream, args, max_over_ranks, barrier)
        gate_cost = gate_leg(K, rank_seed, rank, world, dev, stream, args, max_over_ranks, barrier)

        # Prefix-cache checkpoints every 512 tokens (the pages' hash block) on the same
        # workload: the cost of writing 64 KiB per (checkpoint, head) from the state pass.
        every = 512
        n_ck = K.kda_checkpoint_count(inp["cu_seqlens_host"], every)
        ckbuf = torch.empty(max(n_ck, 1), H, dk, dv, dtype=torch.float32, device=dev)

        def cstep():
            K.kda_prefill_checkpointed(inp["q"], inp["k"], inp["v"], inp["z"], inp["A"], inp["beta"],
                                       inp["cu_seqlens"], inp["cu_seqlens_host"], every,
                                       final_state=S, o=o, checkpoints=ckbuf, workspace=ws,
                                       algo=args.algo, stream=stream)

        for _ in range(args.warmup):
            cstep()
        torch.cuda.synchronize()
        barrier()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            cstep()
        c1.record(stream)
        torch.cuda.synchronize()
        cms = max_over_ranks(c0.elapsed_time(c1), world, dev) / args.steps
        ckpt = {"every": every, "checkpoints_per_step": n_ck * H, "ms_per_step": cms,
                "overhead_vs_plain": cms / ms_per_step - 1.0,
                "extra_bytes_per_step": n_ck * H * dk * dv * 4}
        del ckbuf

        decode = decode_leg(K, rank, world, dev, stream, args, hbm_peak, barrier)

        # End to end through the C ABI: pinned host inputs -> device, prefill, result ->
        # host, every byte of every step inside the timed region.  Steps are
        # pipelined the way a serving loop would run them: two device slots, the
        # host->device copy of step i+1 and the device->host copy of step i on their
        # own streams, overlapping step i's prefill and each other (PCIe is full
        # duplex), so the steady state is bound by the larger copy.
        host = {key: inp[key].cpu().pin_memory() for key in ("q", "k", "v", "z", "beta", "A")}
        host_cu = inp["cu_seqlens_host"].pin_memory()
        dbufs = [{key: torch.empty_like(inp[key]) for key in host} for _ in range(2)]
        cu_devs = [torch.empty_like(inp["cu_seqlens"]) for _ in range(2)]
        o_devs = [o, torch.empty_like(o)]
        S_devs = [S, torch.empty_like(S)]
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        S_host = torch.empty(S.shape, dtype=S.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + host_cu.numel() * 4
        d2h = o_host.numel() * o_host.element_size() + S_host.numel() * 4
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record(stream)

        def e2e_step(i):
            sl = i % 2
            s_in.wait_event(ev_comp[sl])          # slot's inputs were consumed (step i - 2)
            with torch.cuda.stream(s_in):
                for key in host:
                    dbufs[sl][key].copy_(host[key], non_blocking=True)
                cu_devs[sl].copy_(host_cu, non_blocking=True)
            ev_in[sl].record(s_in)
            stream.wait_event(ev_in[sl])
            stream.wait_event(ev_out[sl])         # slot's outputs were read back (step i - 2)
            d = dbufs[sl]
            K.kda_prefill(d["q"], d["k"], d["v"], d["z"], d["A"], d["beta"], cu_devs[sl],
                          inp["cu_seqlens_host"], None, final_state=S_devs[sl], o=o_devs[sl],
                          workspace=ws, algo=args.algo, stream=stream)
            ev_comp[sl].record(stream)
            s_out.wait_event(ev_comp[sl])
            with torch.cuda.stream(s_out):
                o_host.copy_(o_devs[sl], non_blocking=True)
                S_host.copy_(S_devs[sl], non_blocking=True)
            ev_out[sl].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        t1.record(s_out)
        torch.cuda.synchronize()
        ems = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.e2e_steps
        e2e = {"value": tokens / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": args.e2e_steps,
               "pipelining": "2 device slots; host->device, prefill, device->host on 3 streams"}
        del dbufs, cu_devs

        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            r = cpu_oracle_sample(inp, args.cpu_seconds)
            cpu = {"value": r["tokens_per_s"], "unit": "tokens/s", "cores": r["cores"],
                   "kind": "oracle", "sample": r["sample"], "seconds": r["seconds"]}

    in_bytes = sum(inp[key].numel() * inp[key].element_size() for key in ("q", "k", "v", "z"))
    l2_note = (f"{'inputs larger than' if in_bytes > L2_BYTES else 'inputs SMALLER than'} L2 "
               f"(q, k, v, z = {in_bytes / 1e9:.2f} GB per step, L2 {L2_BYTES / 1e6:.0f} MB), no flush")
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": cfg.name, "global_batch": N * world, "seq_len": T, "heads": H,
                       "dk": dk, "dv": dv, "parallelism": f"dp{world} (one independent problem per GPU)",
                       "algo": args.algo,
                       "l2": l2_note},
            "tflops": tflops,
            "roofline": roofline,
            "path_roofline": path,
            "decode": decode,
            "checkpoints": ckpt,
            "sequence_split": split,
            "unbounded_gate": gate_cost,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
