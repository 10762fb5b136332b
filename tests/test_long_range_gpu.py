"""Long-range parity at slow decay (B200 only).

Under the workloads' gate inputs (z ~ N(0, 1)) the per-step decay averages
about e^{-2.5}, so the state forgets within a few tokens and neither the
initial state nor rounding that piles up across chunks shows in the outputs.
With z ~ N(-4, 1) the decay is about 0.93 per step, and with z ~ N(-8, 1) it
is close to 1, so the state carries information across thousands of chunks:
the only limit on memory left is the delta rule's own overwrite along k
("Kimi K3: Architecture, Training, and Million-Token Agentic RL", section 3.1
equation).  These cases exercise the one place where the tensor-core path
rounds its state, the bf16 copy of S that enters the per-chunk products, over
long chains, from a nonzero initial state.  Every element of o and of the
final state is compared with the fp64 oracle (bar 2e-2 for bf16 inputs).
"""
import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import CONFIGS, prefill_inputs
from tests.kda_testutil import TOL_BF16, gpu_subset, oracle_subset, relerr

pytestmark = pytest.mark.gpu


def _cuda(inp):
    return {key: (val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val)
            for key, val in inp.items()}


def _check_every_element(inp, o, S):
    n, H = len(inp["lengths"]), inp["q"].shape[1]
    ref_o, ref_S, tok = oracle_subset(inp, list(range(n)), list(range(H)))
    got_o, got_S = gpu_subset(o, S, tok, list(range(n)), list(range(H)))
    eo, es = relerr(got_o, ref_o), relerr(got_S, ref_S)
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
    return eo, es


@pytest.mark.parametrize("algo", ["tensor_core", "tensor_core_split"])
@pytest.mark.parametrize("z_mean", [-4.0, -8.0])
def test_slow_decay_16k_tokens(algo, z_mean):
    """One 16,384-token sequence (256 chunks), 3 heads, S0 ~ N(0, 0.02^2).
    Forced split: 16 segments of 16 chunks, each composed by the affine scan."""
    L, H = 16384, 3
    x = _cuda(prefill_inputs([L], H, 128, 128, "bf16", seed=40 + int(-z_mean), s0_std=0.02,
                             z_mean=z_mean))
    if algo == "tensor_core_split":
        assert K.kda_prefill_segments(L, 1, H, 128, 128, torch.bfloat16, algo) == 16
    o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=x["initial_state"], algo=algo)
    torch.cuda.synchronize()
    assert K.kda_device_status() == 0
    _check_every_element(x, o, S)


@pytest.mark.parametrize("algo", ["tensor_core", "tensor_core_split"])
def test_slow_decay_varlen_resume_lengths(algo):
    """The 16 packed sequence lengths of the varlen prefix-resume workload
    (log-uniform in [1K, 64K], about 248K tokens) at 2 heads, slow decay,
    nonzero initial states, final states written."""
    lengths = CONFIGS["varlen_resume"].lengths
    x = _cuda(prefill_inputs(lengths, 2, 128, 128, "bf16", seed=43, s0_std=0.02, z_mean=-4.0))
    o, S = K.kda_prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=x["initial_state"], algo=algo)
    torch.cuda.synchronize()
    assert K.kda_device_status() == 0
    _check_every_element(x, o, S)
