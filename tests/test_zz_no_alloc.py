"""kda_prefill_noalloc against kda_prefill (B200 only).

The no-allocation entry point serves callers that cannot allocate device
memory at call time; it keeps its scratch in one fixed device array that every
call shares.  Two calls in a row with different inputs must each match the
regular entry point (which takes a caller-allocated workspace) within the
bf16 parity tolerance -- the second call must not see the first one's leftovers.
This file is named so that pytest collects it last.
"""
import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import prefill_inputs
from tests.kda_testutil import TOL_BF16, relerr, to_np

pytestmark = pytest.mark.gpu


def _on_gpu(x):
    return {key: (val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val)
            for key, val in x.items()}


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [prefill_inputs([200, 0, 77, 64], 3, 128, 128, "bf16", seed=21, s0_std=0.02),
             prefill_inputs([33, 150], 4, 128, 128, "bf16", seed=22, s0_std=0.05)]
    for x in cases:
        x = _on_gpu(x)
        args = (x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
                x["cu_seqlens_host"])
        o_ref, s_ref = K.kda_prefill(*args, initial_state=x["initial_state"])
        o_na, s_na = K.kda_prefill_noalloc(*args, initial_state=x["initial_state"])
        torch.cuda.synchronize()
        assert relerr(to_np(o_na), to_np(o_ref)) <= TOL_BF16
        assert relerr(to_np(s_na), to_np(s_ref)) <= TOL_BF16
    assert K.kda_device_status() == 0
