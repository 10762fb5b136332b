"""GPU parity: the CUDA library against the fp64 CPU oracle (B200 only).

Metric: max|err| / max|ref| per output tensor (o and final state separately);
bar 2e-2 for bf16 inputs with fp32 state, 1e-4 for fp32 inputs.  Every call
goes through the C ABI (ctypes binding).  Full-size workloads are compared on
sampled (sequence, head) pairs, each computed whole by the oracle.
"""
import numpy as np
import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import (CONFIGS, config_inputs,
                                                             decode_inputs, prefill_inputs)
from oracle import oracle
from tests.kda_testutil import (TOL_BF16, TOL_F32, gpu_subset, oracle_subset, relerr, to_np)

pytestmark = pytest.mark.gpu

# tensor_core_split forces the affine-scan split of every sequence into >= 2
# segments (one segment per chunk for sequences shorter than that).
PREFILL_ALGOS = ["cuda_core", "tensor_core", "tensor_core_split"]


def _supported(algo, dtype="bf16", dk=128, dv=128):
    if algo.startswith("tensor_core") and (dtype != "bf16" or dk != 128 or dv != 128):
        pytest.skip("the tensor-core path covers bf16 with dk = dv = 128")


def _cuda(inp):
    out = {}
    for key, val in inp.items():
        out[key] = val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val
    return out


def _run(inp, algo="auto", **kw):
    return K.kda_prefill(inp["q"], inp["k"], inp["v"], inp["z"], inp["A"], inp["beta"],
                         inp["cu_seqlens"], inp["cu_seqlens_host"],
                         initial_state=inp["initial_state"], algo=algo, **kw)


def _check_all(inp, o, S, tol):
    n = len(inp["lengths"])
    ref_o, ref_S, tok = oracle_subset(inp, list(range(n)), list(range(inp["q"].shape[1])))
    got_o, got_S = gpu_subset(o, S, tok, list(range(n)), list(range(inp["q"].shape[1])))
    eo, es = relerr(got_o, ref_o) if got_o.size else 0.0, relerr(got_S, ref_S)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


def test_tiny_f32_config():
    inp = _cuda(config_inputs(CONFIGS["tiny_f32"]))
    o, S = _run(inp)
    torch.cuda.synchronize()
    _check_all(inp, o, S, TOL_F32)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 128), (128, 32)])
def test_ragged_varlen_small(algo, dtype, dk, dv):
    _supported(algo, dtype, dk, dv)
    lengths = [1, 15, 16, 17, 100, 0, 257, 64]
    inp = _cuda(prefill_inputs(lengths, 3, dk, dv, dtype, seed=dk + dv, s0_std=0.02))
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    _check_all(inp, o, S, TOL_F32 if dtype == "f32" else TOL_BF16)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_prefill_4k_full(algo):
    inp = _cuda(config_inputs(CONFIGS["prefill_4k"]))
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    _check_all(inp, o, S, TOL_BF16)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_prefill_32k_sampled_heads(algo):
    cfg = CONFIGS["prefill_32k"]
    inp = config_inputs(cfg, device="cuda")
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    heads = [0, 47, 95]
    ref_o, ref_S, tok = oracle_subset(inp, [0], heads)
    got_o, got_S = gpu_subset(o, S, tok, [0], heads)
    assert relerr(got_o, ref_o) <= TOL_BF16
    assert relerr(got_S, ref_S) <= TOL_BF16
    assert torch.isfinite(o).all()


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_varlen_resume_sampled(algo):
    cfg = CONFIGS["varlen_resume"]
    inp = config_inputs(cfg, device="cuda")
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    lens = inp["lengths"]
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 5})
    heads = [0, 95]
    ref_o, ref_S, tok = oracle_subset(inp, seqs, heads)
    got_o, got_S = gpu_subset(o, S, tok, seqs, heads)
    assert relerr(got_o, ref_o) <= TOL_BF16
    assert relerr(got_S, ref_S) <= TOL_BF16
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
@pytest.mark.parametrize("case", ["saturated", "alpha_one_beta_one", "slow_decay"])
def test_gate_edge_cases(algo, case):
    lengths = [48, 17, 33]
    kw = dict(saturated=dict(z_mean=1e4, z_std=0.0),
              alpha_one_beta_one=dict(z_mean=-1e4, z_std=0.0, beta_value=1.0),
              slow_decay=dict(z_mean=-4.0))[case]
    inp = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=7, s0_std=0.02, **kw))
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    _check_all(inp, o, S, TOL_BF16)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_empty_sequences_pass_state_through(algo):
    lengths = [0, 0, 5, 0, 40]
    inp = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=8, s0_std=0.5))
    o, S = _run(inp, algo)
    torch.cuda.synchronize()
    for n in (0, 1, 3):
        assert torch.equal(S[n], inp["initial_state"][n])
    _check_all(inp, o, S, TOL_BF16)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_in_place_resume_and_split_equivalence(algo):
    """Prefix-cache resume: prefill(x[:t1]) -> S, then prefill(x[t1:], S0 = S)
    with final_state aliasing initial_state, equals prefill(x)."""
    L = 300
    full = _cuda(prefill_inputs([L], 2, 128, 128, "bf16", seed=9, s0_std=0.02))
    o_full, S_full = _run(full, algo)
    for t1 in (16, 77, 128):
        def part(lo, hi, s0):
            d = {key: full[key][lo:hi] for key in ("q", "k", "v", "z", "beta")}
            cu = torch.tensor([0, hi - lo], dtype=torch.int32)
            return dict(d, A=full["A"], cu_seqlens=cu.cuda(), cu_seqlens_host=cu,
                        initial_state=s0, lengths=[hi - lo])
        a = part(0, t1, full["initial_state"].clone())
        oa, sa = _run(a, algo, final_state=a["initial_state"])
        assert sa.data_ptr() == a["initial_state"].data_ptr()
        b = part(t1, L, sa)
        ob, sb = _run(b, algo, final_state=sa)
        torch.cuda.synchronize()
        assert relerr(to_np(torch.cat([oa, ob])), to_np(o_full)) <= TOL_BF16
        assert relerr(to_np(sb), to_np(S_full)) <= TOL_BF16
    _check_all(full, o_full, S_full, TOL_BF16)


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_outputs_stay_inside_their_buffers(algo):
    """Guard regions around o and the final state are left untouched."""
    lengths = [5, 31, 16, 70]
    inp = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=10))
    T, H, dv, dk, N = sum(lengths), 2, 128, 128, 4
    guard = 4096
    obuf = torch.full((guard * 2 + T * H * dv,), 7.0, dtype=torch.bfloat16, device="cuda")
    sbuf = torch.full((guard * 2 + N * H * dk * dv,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[guard:guard + T * H * dv].view(T, H, dv)
    S = sbuf[guard:guard + N * H * dk * dv].view(N, H, dk, dv)
    _run(inp, algo, o=o, final_state=S)
    torch.cuda.synchronize()
    assert torch.all(obuf[:guard] == 7.0) and torch.all(obuf[-guard:] == 7.0)
    assert torch.all(sbuf[:guard] == 7.0) and torch.all(sbuf[-guard:] == 7.0)
    _check_all(inp, o, S, TOL_BF16)


# ---------------------------------------------------------- sequence split ----

def test_split_long_single_head_sequence_sixteen_segments():
    """One head, one 3,109-token sequence (49 chunks) cut into 16 segments of 3
    or 4 chunks with a ragged tail, from a nonzero initial state: outputs and
    final state against the oracle, and against the unsplit tensor-core path."""
    L, H = 3109, 1
    x = _cuda(prefill_inputs([L], H, 128, 128, "bf16", seed=31, s0_std=0.02))
    assert K.kda_prefill_segments(L, 1, H, 128, 128, torch.bfloat16, "tensor_core_split") == 16
    assert K.kda_prefill_segments(L, 1, H, 128, 128, torch.bfloat16, "auto") == 3
    o, S = _run(x, "tensor_core_split")
    o1, S1 = _run(x, "tensor_core")
    torch.cuda.synchronize()
    _check_all(x, o, S, TOL_BF16)
    assert relerr(to_np(o), to_np(o1)) <= TOL_BF16
    assert relerr(to_np(S), to_np(S1)) <= TOL_BF16


@pytest.mark.parametrize("lengths,H", [([64 * 33], 4), ([130, 64 * 20 + 5, 64], 3), ([63 * 64 + 1], 2)])
def test_split_segment_boundaries(lengths, H):
    """Segment edges on and off chunk boundaries, a one-chunk sequence next to
    split ones, and a one-token last chunk."""
    x = _cuda(prefill_inputs(lengths, H, 128, 128, "bf16", seed=sum(lengths) + H, s0_std=0.05))
    o, S = _run(x, "tensor_core_split")
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    _check_all(x, o, S, TOL_BF16)


def test_auto_splits_the_4k_single_sequence_and_records_five_kernels():
    """AUTO picks 2 segments for 32 heads x 4,096 tokens, launches 5 kernels
    (one event boundary each) and gives the forced split's result bit for bit."""
    cfg = CONFIGS["prefill_4k"]
    x = config_inputs(cfg, device="cuda")
    T = x["q"].shape[0]
    assert K.kda_prefill_segments(T, 1, cfg.H, 128, 128, torch.bfloat16, "auto") == 2
    assert K.kda_prefill_kernel_count(T, 1, cfg.H, 128, 128, torch.bfloat16, "auto") == 5
    assert K.kda_prefill_kernel_count(T, 1, cfg.H, 128, 128, torch.bfloat16, "tensor_core") == 3
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in evs:
        e.record()  # torch creates the CUDA event at its first record
    o, S = _run(x, "auto", stage_events=evs)
    o2, S2 = _run(x, "tensor_core_split")
    torch.cuda.synchronize()
    assert all(evs[i].elapsed_time(evs[i + 1]) >= 0 for i in range(5))
    assert torch.equal(o, o2) and torch.equal(S, S2)


def test_auto_with_checkpoints_keeps_sequences_whole():
    """Checkpoints come from the unsplit chain: AUTO on a split-eligible shape
    with checkpoints equals the forced unsplit path, and the oracle."""
    L, H = 64 * 40, 8
    x = _cuda(prefill_inputs([L], H, 128, 128, "bf16", seed=33, s0_std=0.02))
    assert K.kda_prefill_segments(L, 1, H, 128, 128, torch.bfloat16, "auto") == 2
    got = K.kda_prefill_checkpointed(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                     x["cu_seqlens"], x["cu_seqlens_host"], 512,
                                     initial_state=x["initial_state"], algo="auto")
    ref = K.kda_prefill_checkpointed(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                     x["cu_seqlens"], x["cu_seqlens_host"], 512,
                                     initial_state=x["initial_state"], algo="tensor_core")
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    _, ref_S, ref_ck = oracle.prefill_checkpoints(
        x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens_host"], 512,
        x["initial_state"])
    assert relerr(to_np(got[2]), ref_ck) <= TOL_BF16
    assert relerr(to_np(got[1]), ref_S) <= TOL_BF16


# ------------------------------------------------ stage intermediates ----

def test_stage_intermediates_match_the_chunkwise_form():
    """The debug entry point's dumps of the fused stages, each against the fp64
    chunkwise form at the tensor-core path's 64-token chunks: a1 G (fp32), a2 W
    and U, a3 delta = U - W S_in (bf16 values) -- and the dumps change nothing."""
    from oracle import chunkwise
    lengths = [1, 63, 64, 65, 130, 200]
    x = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=90, s0_std=0.05))
    d = K.kda_prefill_debug(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                            x["cu_seqlens_host"], initial_state=x["initial_state"])
    o_plain, S_plain = _run(x, "tensor_core")
    torch.cuda.synchronize()
    assert torch.equal(d["o"], o_plain) and torch.equal(d["final_state"], S_plain)
    ref = chunkwise.prefill_intermediates(*(to_np(x[key]) for key in ("q", "k", "v", "z", "A", "beta")),
                                          x["cu_seqlens_host"].numpy(), to_np(x["initial_state"]), chunk=64)
    for key, dkey, tol in (("G", "G", 1e-5), ("W", "W", TOL_BF16), ("U", "U", TOL_BF16),
                           ("delta", "D", TOL_BF16)):
        got = to_np(d[key])
        assert np.isfinite(got).all(), key
        assert relerr(got, ref[dkey]) <= tol, (key, relerr(got, ref[dkey]))
    assert relerr(to_np(d["o"]), ref["o"]) <= TOL_BF16
    assert relerr(to_np(d["final_state"]), ref["final_state"]) <= TOL_BF16


# ------------------------------------------------------- plan edge cases ----

@pytest.mark.parametrize("algo", ["tensor_core", "tensor_core_split"])
def test_more_sequences_than_the_sorted_plan(algo):
    """4,200 sequences of 0-70 tokens: above the 4,096 sequences the plan sorts
    longest-first, so launch order falls back to the identity; every output and
    final state against the oracle."""
    rs = np.random.RandomState(80)
    lengths = [int(x) for x in rs.randint(0, 71, size=4200)]
    x = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=81, s0_std=0.02))
    o, S = _run(x, algo)
    torch.cuda.synchronize()
    _check_all(x, o, S, TOL_BF16)


@pytest.mark.parametrize("algo", ["tensor_core", "tensor_core_split"])
def test_one_long_sequence_two_heads(algo):
    """65,537 tokens (1,025 chunks, a one-token last chunk), 2 heads: the whole
    chain, and 16 segments of 64-65 chunks, against the oracle."""
    L = 65537
    x = _cuda(prefill_inputs([L], 2, 128, 128, "bf16", seed=82, s0_std=0.02))
    if algo == "tensor_core_split":
        assert K.kda_prefill_segments(L, 1, 2, 128, 128, torch.bfloat16, algo) == 16
    o, S = _run(x, algo)
    torch.cuda.synchronize()
    _check_all(x, o, S, TOL_BF16)


def test_split_with_empty_and_single_chunk_sequences_interleaved():
    lengths = [0, 64 * 9 + 3, 0, 1, 64 * 5, 0]
    x = _cuda(prefill_inputs(lengths, 3, 128, 128, "bf16", seed=83, s0_std=0.3))
    o, S = _run(x, "tensor_core_split")
    torch.cuda.synchronize()
    for n in (0, 2, 5):
        assert torch.equal(S[n], x["initial_state"][n])
    _check_all(x, o, S, TOL_BF16)


# ------------------------------------------------- unbounded (Softplus) gate ----

@pytest.mark.parametrize("algo,dtype,tol", [("cuda_core", "f32", TOL_F32), ("cuda_core", "bf16", TOL_BF16),
                                            ("tensor_core", "bf16", TOL_BF16),
                                            ("tensor_core_split", "bf16", TOL_BF16)])
@pytest.mark.parametrize("z_mean", [0.0, 3.0])
def test_softplus_gate_prefill_matches_oracle(algo, dtype, tol, z_mean):
    """The unbounded gate: on the CUDA-core path (every 16-token chunk pair by
    pair) and on the tensor-core path (off-diagonal sub-tile pairs on tcgen05,
    the diagonal 16 x 16 tiles pair by pair).  At z_mean = 3 a 16-token
    cumulative log-decay reaches well below -88, where the dense tile form's
    e^{-G} would overflow fp32."""
    lengths = [1, 15, 16, 17, 100, 0, 257]
    x = _cuda(prefill_inputs(lengths, 3, 128, 128, dtype, seed=70 + int(z_mean), s0_std=0.02,
                             z_mean=z_mean))
    if z_mean > 0:
        from oracle import oracle as orc
        g = orc.gate(x["z"], x["A"], "softplus")
        # tokens 165..180: one 16-token chunk of the 257-token sequence (starts at 149)
        assert np.cumsum(g[165:181], axis=0).min() < -88.0
    o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=x["initial_state"], gate="softplus",
                         algo=algo)
    torch.cuda.synchronize()
    assert K.kda_device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    n, H = len(lengths), 3
    ref_o, ref_S, tok = oracle_subset(x, list(range(n)), list(range(H)), gate="softplus")
    got_o, got_S = gpu_subset(o, S, tok, list(range(n)), list(range(H)))
    assert relerr(got_o, ref_o) <= tol and relerr(got_S, ref_S) <= tol


@pytest.mark.parametrize("algo", ["cuda_core", "tensor_core"])
def test_softplus_gate_saturated_decay(algo):
    """z = 60: per-token log-decay far below the -110 clamp, the state is wiped
    at every step; both sides agree and nothing overflows."""
    x = _cuda(prefill_inputs([70, 33], 2, 128, 128, "bf16", seed=72, s0_std=0.5, z_mean=60.0,
                             z_std=0.0))
    o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=x["initial_state"], gate="softplus",
                         algo=algo)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    ref_o, ref_S, tok = oracle_subset(x, [0, 1], [0, 1], gate="softplus")
    got_o, got_S = gpu_subset(o, S, tok, [0, 1], [0, 1])
    assert relerr(got_o, ref_o) <= TOL_BF16 and relerr(got_S, ref_S) <= TOL_BF16


def test_softplus_gate_bounded_inputs_differ_from_bounded_gate():
    """The gate selector is live: the same inputs under the two gates differ,
    and the bounded call through the gated entry point equals kda_prefill."""
    x = _cuda(prefill_inputs([80], 2, 128, 128, "f32", seed=73))
    o_b, S_b = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                             x["cu_seqlens_host"], algo="cuda_core")
    o_s, _ = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                           x["cu_seqlens_host"], algo="cuda_core", gate="softplus")
    ws = torch.empty(0, dtype=torch.uint8, device="cuda")
    o_g = torch.empty_like(o_b)
    S_g = torch.empty_like(S_b)
    ch = x["cu_seqlens_host"].to(torch.int32).contiguous()
    code = K._lib.kda_prefill_gated(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["z"].data_ptr(), x["A"].data_ptr(),
        x["beta"].data_ptr(), x["cu_seqlens"].data_ptr(), ch.data_ptr(), 1, 80, 2, 128, 128, 1,
        None, S_g.data_ptr(), o_g.data_ptr(), None, 0, K.KDA_ALGO["cuda_core"], 0, None)
    torch.cuda.synchronize()
    assert code == 0
    assert torch.equal(o_g, o_b) and torch.equal(S_g, S_b)
    assert (o_s - o_b).abs().max().item() > 1e-3


def test_softplus_gate_tensor_core_long_sequence_sampled_heads():
    """The unbounded gate's tensor-core path on 4,096 tokens x 8 heads at the
    workload distributions (every element of o and S), and its agreement with
    the bounded gate's path when the Softplus decay is mild enough that both
    read the same inputs differently (the selector is live)."""
    x = _cuda(prefill_inputs([4096], 8, 128, 128, "bf16", seed=75, s0_std=0.02))
    o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=x["initial_state"], gate="softplus",
                         algo="tensor_core")
    ob, _ = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                          x["cu_seqlens_host"], initial_state=x["initial_state"], algo="tensor_core")
    torch.cuda.synchronize()
    assert K.kda_device_status() == 0
    ref_o, ref_S, tok = oracle_subset(x, [0], list(range(8)), gate="softplus")
    got_o, got_S = gpu_subset(o, S, tok, [0], list(range(8)))
    assert relerr(got_o, ref_o) <= TOL_BF16 and relerr(got_S, ref_S) <= TOL_BF16
    assert (o.float() - ob.float()).abs().max().item() > 1e-2


@pytest.mark.parametrize("dtype,tol", [("f32", TOL_F32), ("bf16", TOL_BF16)])
def test_softplus_gate_decode_matches_oracle(dtype, tol):
    d = decode_inputs(16, 4, 128, 128, dtype, seed=74, nsets=2, device="cuda")
    st = d["state"].clone()
    o = K.kda_decode_step(d["q"][0], d["k"][0], d["v"][0], d["z"][0], d["A"], d["beta"][0], st,
                          gate="softplus")
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.decode_step(d["q"][0], d["k"][0], d["v"][0], d["z"][0], d["A"],
                                      d["beta"][0], d["state"], gate="softplus")
    assert relerr(to_np(o), ref_o) <= tol and relerr(to_np(st), ref_S) <= tol


# ------------------------------------------------------------------ decode ----

@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("f32", TOL_F32)])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128)])
def test_decode_step_with_slots(dtype, tol, dk, dv):
    B, H, P = 37, 3, 50
    d = decode_inputs(B, H, dk, dv, dtype, seed=11, nsets=2, pool=P, permute_slots=True,
                      device="cuda")
    pool0 = d["state"].clone()
    o = K.kda_decode_step(d["q"][0], d["k"][0], d["v"][0], d["z"][0], d["A"], d["beta"][0],
                          d["state"], d["slots"])
    torch.cuda.synchronize()
    ref_o, ref_new = oracle.decode_step(d["q"][0], d["k"][0], d["v"][0], d["z"][0], d["A"],
                                        d["beta"][0], pool0, d["slots"])
    assert relerr(to_np(o), ref_o) <= tol
    assert relerr(to_np(d["state"]), ref_new) <= tol
    untouched = sorted(set(range(P)) - set(d["slots"].cpu().tolist()))
    assert torch.equal(d["state"][untouched], pool0[untouched])


def test_decode_full_batch_first_steps():
    cfg = CONFIGS["decode_256"]
    d = decode_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.dtype, seed=cfg.seed, nsets=cfg.nsets,
                      device="cuda")
    ref_state = to_np(d["state"])
    for s in range(2):
        o = K.kda_decode_step(d["q"][s], d["k"][s], d["v"][s], d["z"][s], d["A"], d["beta"][s],
                              d["state"])
        torch.cuda.synchronize()
        ref_o, ref_state = oracle.decode_step(d["q"][s], d["k"][s], d["v"][s], d["z"][s], d["A"],
                                              d["beta"][s], ref_state)
        assert relerr(to_np(o), ref_o) <= TOL_BF16
        assert relerr(to_np(d["state"]), ref_state) <= TOL_BF16


def test_decode_1000_steps_sampled_pairs():
    """The timed decode workload: 1000 in-place steps (step s uses input set
    s mod 16); sampled (sequence, head) pairs are replayed by the oracle."""
    cfg = CONFIGS["decode_256"]
    d = decode_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, cfg.dtype, seed=cfg.seed, nsets=cfg.nsets,
                      device="cuda")
    bsel, hsel = np.array([0, 101, 255]), np.array([0, 50, 95])
    ref_state = to_np(d["state"])[bsel][:, hsel]
    subsets = [{key: to_np(d[key][i])[bsel][:, hsel] for key in ("q", "k", "v", "z", "beta")}
               for i in range(cfg.nsets)]
    A_sub = to_np(d["A"])[hsel]
    for s in range(cfg.steps):
        i = s % cfg.nsets
        o = K.kda_decode_step(d["q"][i], d["k"][i], d["v"][i], d["z"][i], d["A"], d["beta"][i],
                              d["state"])
        sub = subsets[i]
        ref_o, ref_state = oracle.decode_step(sub["q"], sub["k"], sub["v"], sub["z"], A_sub,
                                              sub["beta"], ref_state)
    torch.cuda.synchronize()
    got_o = to_np(o)[bsel][:, hsel]
    got_S = to_np(d["state"])[bsel][:, hsel]
    assert relerr(got_o, ref_o) <= TOL_BF16
    assert relerr(got_S, ref_state) <= TOL_BF16


@pytest.mark.parametrize("algo", PREFILL_ALGOS)
def test_prefill_then_decode_equals_longer_prefill(algo):
    L = 70
    full = _cuda(prefill_inputs([L + 1], 3, 128, 128, "bf16", seed=12, s0_std=0.02))
    o_full, S_full = _run(full, algo)
    head = {key: full[key][:L] for key in ("q", "k", "v", "z", "beta")}
    cu = torch.tensor([0, L], dtype=torch.int32)
    _, S = _run(dict(head, A=full["A"], cu_seqlens=cu.cuda(), cu_seqlens_host=cu,
                     initial_state=full["initial_state"], lengths=[L]), algo)
    o = K.kda_decode_step(*(full[key][L:L + 1].contiguous() for key in ("q", "k", "v", "z")),
                          full["A"], full["beta"][L:L + 1].contiguous(), S)
    torch.cuda.synchronize()
    assert relerr(to_np(o[0]), to_np(o_full[L])) <= TOL_BF16
    assert relerr(to_np(S), to_np(S_full)) <= TOL_BF16


# ------------------------------------------------------------- checkpoints ----

@pytest.mark.parametrize("algo,dtype,tol", [("cuda_core", "f32", TOL_F32), ("cuda_core", "bf16", TOL_BF16),
                                            ("tensor_core", "bf16", TOL_BF16)])
@pytest.mark.parametrize("every", [64, 128, 512])
def test_checkpoints_match_oracle(algo, dtype, tol, every):
    """State checkpoints every `every` tokens (prefix-cache boundaries) equal the
    oracle's, and asking for them leaves o and the final states unchanged."""
    lengths = [700, 64, 129, 0, 1030, 511]
    x = _cuda(prefill_inputs(lengths, 2, 128, 128, dtype, seed=50 + every, s0_std=0.02))
    o, S, ck = K.kda_prefill_checkpointed(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                          x["cu_seqlens"], x["cu_seqlens_host"], every,
                                          initial_state=x["initial_state"], algo=algo)
    o2, S2 = _run(x, algo)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(S, S2)
    ref_o, ref_S, ref_ck = oracle.prefill_checkpoints(
        x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens_host"], every,
        x["initial_state"])
    assert ck.shape[0] == sum(L // every for L in lengths) == ref_ck.shape[0]
    assert relerr(to_np(ck), ref_ck) <= tol
    assert relerr(to_np(S), ref_S) <= tol


def test_checkpoints_full_size_varlen_sampled_heads():
    """The 16-sequence varlen workload with checkpoints every 512 tokens (the
    pages' prefix-hash block); two heads of every checkpoint row against the oracle."""
    cfg = CONFIGS["varlen_resume"]
    x = config_inputs(cfg, device="cuda")
    o, S, ck = K.kda_prefill_checkpointed(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                          x["cu_seqlens"], x["cu_seqlens_host"], 512,
                                          initial_state=x["initial_state"])
    torch.cuda.synchronize()
    heads = [0, 77]
    hs = torch.tensor(heads, device="cuda")
    sub = {key: x[key].index_select(1, hs).cpu() for key in ("q", "k", "v", "z", "beta")}
    _, ref_S, ref_ck = oracle.prefill_checkpoints(sub["q"], sub["k"], sub["v"], sub["z"],
                                                  x["A"].index_select(0, hs).cpu(), sub["beta"],
                                                  x["cu_seqlens_host"], 512,
                                                  x["initial_state"].index_select(1, hs).cpu())
    assert relerr(to_np(ck.index_select(1, hs)), ref_ck) <= TOL_BF16
    assert relerr(to_np(S.index_select(1, hs)), ref_S) <= TOL_BF16


# ---------------------------------------------- speculative verify / replay ----

def _spec_inputs(B, Tq, H, dk, dv, dtype, seed, pool):
    x = prefill_inputs([Tq] * B, H, dk, dv, dtype, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    state = (torch.randn(pool, H, dk, dv, generator=g) * 0.3).cuda()
    slots = torch.randperm(pool, generator=g)[:B].to(torch.int32).cuda()
    shaped = {key: x[key].view(B, Tq, *x[key].shape[1:]).cuda() for key in ("q", "k", "v", "z", "beta")}
    return x, shaped, state, slots


@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("f32", TOL_F32)])
def test_spec_verify_leaves_state_and_matches_prefill(dtype, tol):
    B, Tq, H, dk, dv, P = 37, 5, 3, 128, 128, 50
    x, s, state, slots = _spec_inputs(B, Tq, H, dk, dv, dtype, 60, P)
    before = state.clone()
    o = K.kda_decode_multi(s["q"], s["k"], s["v"], s["z"], x["A"].cuda(), s["beta"], state, slots)
    torch.cuda.synchronize()
    assert torch.equal(state, before)                      # a verify writes no state
    s0 = before[slots.long()].cpu()
    ref_o, _ = oracle.prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens_host"], s0)
    assert relerr(to_np(o).reshape(B * Tq, H, dv), ref_o) <= tol


@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("f32", TOL_F32)])
def test_spec_replay_commits_accepted_prefix(dtype, tol):
    B, Tq, H, dk, dv, P = 37, 6, 3, 64, 128, 41
    x, s, state, slots = _spec_inputs(B, Tq, H, dk, dv, dtype, 61, P)
    before = state.clone()
    g = torch.Generator().manual_seed(7)
    acc = torch.randint(0, Tq + 1, (B,), generator=g).to(torch.int32)
    acc[0], acc[1] = 0, Tq
    K.kda_decode_multi(s["q"], s["k"], s["v"], s["z"], x["A"].cuda(), s["beta"], state, slots,
                       num_tokens=acc.cuda(), update_state=True, want_outputs=False)
    torch.cuda.synchronize()
    sl = slots.long().cpu()
    untouched = sorted(set(range(P)) - set(sl.tolist()))
    assert torch.equal(state[untouched], before[untouched])
    assert torch.equal(state[sl[0]], before[sl[0]])         # zero accepted tokens: unchanged
    for b in range(B):
        a = int(acc[b])
        if a == 0:
            continue
        tok = slice(b * Tq, b * Tq + a)
        _, ref_S = oracle.prefill(*(x[key][tok] for key in ("q", "k", "v", "z")), x["A"],
                                  x["beta"][tok], np.array([0, a], np.int32),
                                  before[sl[b]].cpu()[None])
        assert relerr(to_np(state[sl[b]]), ref_S[0]) <= tol


def test_spec_single_token_replay_equals_decode_step():
    B, H = 16, 4
    d = decode_inputs(B, H, 128, 128, "bf16", seed=62, nsets=1, device="cuda")
    st1, st2 = d["state"].clone(), d["state"].clone()
    o1 = K.kda_decode_step(d["q"][0], d["k"][0], d["v"][0], d["z"][0], d["A"], d["beta"][0], st1)
    o2 = K.kda_decode_multi(d["q"][0][:, None], d["k"][0][:, None], d["v"][0][:, None],
                            d["z"][0][:, None], d["A"], d["beta"][0][:, None], st2,
                            update_state=True)
    torch.cuda.synchronize()
    assert torch.equal(st1, st2)
    assert torch.equal(o1, o2[:, 0])


def test_spec_full_batch_verify_then_replay():
    """B = 256 sequences, H = 96, 4 drafts each: verify, then replay all four,
    equals four decode steps; the verify outputs equal the steps' outputs."""
    B, H, Tq = 256, 96, 4
    d = decode_inputs(B, H, 128, 128, "bf16", seed=63, nsets=Tq, device="cuda")
    q, k, v, z = (d[key].permute(1, 0, 2, 3).contiguous() for key in ("q", "k", "v", "z"))
    beta = d["beta"].permute(1, 0, 2).contiguous()
    st_steps = d["state"].clone()
    outs = [K.kda_decode_step(d["q"][t], d["k"][t], d["v"][t], d["z"][t], d["A"], d["beta"][t], st_steps)
            for t in range(Tq)]
    st = d["state"].clone()
    ov = K.kda_decode_multi(q, k, v, z, d["A"], beta, st)
    K.kda_decode_multi(q, k, v, z, d["A"], beta, st, update_state=True, want_outputs=False)
    torch.cuda.synchronize()
    assert relerr(to_np(st), to_np(st_steps)) <= 1e-6
    for t in range(Tq):
        assert relerr(to_np(ov[:, t]), to_np(outs[t])) <= 1e-2


@pytest.mark.parametrize("dk,dv,B", [(128, 128, 100), (64, 32, 1300)])
def test_spec_persistent_ctas_two_groups(dk, dv, B):
    """More (sequence, head) items than resident CTAs, so every CTA walks several
    items (state copy and first-group prefetch of the next item during the
    current one), with 11 drafts (a second token group fetched from global
    memory), random slots and accepted counts including 0 and all: verify
    outputs and replayed states against the oracle."""
    H, Tq = 4, 11
    P = B + 7
    x, s, state, slots = _spec_inputs(B, Tq, H, dk, dv, "bf16", 64 + dk, P)
    before = state.clone()
    o = K.kda_decode_multi(s["q"], s["k"], s["v"], s["z"], x["A"].cuda(), s["beta"], state, slots)
    torch.cuda.synchronize()
    assert torch.equal(state, before)
    s0 = before[slots.long()].cpu()
    ref_o, _ = oracle.prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens_host"], s0)
    assert relerr(to_np(o).reshape(B * Tq, H, dv), ref_o) <= TOL_BF16

    g = torch.Generator().manual_seed(dk + dv)
    acc = torch.randint(0, Tq + 1, (B,), generator=g).to(torch.int32)
    acc[0], acc[1], acc[2] = 0, Tq, 8
    K.kda_decode_multi(s["q"], s["k"], s["v"], s["z"], x["A"].cuda(), s["beta"], state, slots,
                       num_tokens=acc.cuda(), update_state=True, want_outputs=False)
    torch.cuda.synchronize()
    sl = slots.long().cpu()
    untouched = sorted(set(range(P)) - set(sl.tolist()))
    assert torch.equal(state[untouched], before[untouched])
    for b in list(range(6)) + list(range(B - 3, B)):
        a = int(acc[b])
        if a == 0:
            assert torch.equal(state[sl[b]], before[sl[b]])
            continue
        tok = slice(b * Tq, b * Tq + a)
        _, ref_S = oracle.prefill(*(x[key][tok] for key in ("q", "k", "v", "z")), x["A"],
                                  x["beta"][tok], np.array([0, a], np.int32),
                                  before[sl[b]].cpu()[None])
        assert relerr(to_np(state[sl[b]]), ref_S[0]) <= TOL_BF16
