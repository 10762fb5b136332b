"""kda_prefill_noalloc against the oracle and against kda_prefill (B200 only).

Some callers cannot allocate device memory when they call the mixer: a serving
engine that hands all free HBM to its paged cache pool at start-up and forbids
later allocations, or code that runs under another framework's allocator.  The
no-allocation entry point takes no workspace; its scratch is one fixed 64 MiB
device array that every call on a device shares.

* Two calls in a row with different inputs must each match the oracle and the
  regular entry point (which takes a caller-allocated workspace) within the
  bf16 parity tolerance: the second call must not see the first one's leftovers.
  Each case runs kda_prefill first, so in a fresh process the first no-alloc
  call -- the one that places the array in device memory, since the runtime
  loads device code lazily -- comes after other device work.
* A call whose workspace is just under the 64 MiB limit (one 576-token sequence
  at 96 heads) runs and matches too.

This file is named so that pytest collects it last.
"""
import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import prefill_inputs
from tests.kda_testutil import TOL_BF16, gpu_subset, oracle_subset, relerr, to_np

pytestmark = pytest.mark.gpu


def _on_gpu(x):
    return {key: (val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val)
            for key, val in x.items()}


def _check(x, o_na, s_na, o_ref, s_ref):
    n, H = len(x["lengths"]), x["q"].shape[1]
    ref_o, ref_S, tok = oracle_subset(x, list(range(n)), list(range(H)))
    got_o, got_S = gpu_subset(o_na, s_na, tok, list(range(n)), list(range(H)))
    assert relerr(got_o, ref_o) <= TOL_BF16
    assert relerr(got_S, ref_S) <= TOL_BF16
    assert relerr(to_np(o_na), to_np(o_ref)) <= TOL_BF16
    assert relerr(to_np(s_na), to_np(s_ref)) <= TOL_BF16


def _both(x):
    args = (x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"], x["cu_seqlens"],
            x["cu_seqlens_host"])
    o_ref, s_ref = K.kda_prefill(*args, initial_state=x["initial_state"])
    o_na, s_na = K.kda_prefill_noalloc(*args, initial_state=x["initial_state"])
    torch.cuda.synchronize()
    return o_na, s_na, o_ref, s_ref


def test_noalloc_matches_oracle_and_workspace_entry_point_twice():
    cases = [prefill_inputs([200, 0, 77, 64], 3, 128, 128, "bf16", seed=21, s0_std=0.02),
             prefill_inputs([33, 150], 4, 128, 128, "bf16", seed=22, s0_std=0.05)]
    for x in cases:
        x = _on_gpu(x)
        _check(x, *_both(x))
    assert K.kda_device_status() == 0


def test_noalloc_just_under_the_scratch_limit():
    limit = 64 << 20
    assert K.kda_prefill_workspace_size(576, 1, 96, 128, 128, torch.bfloat16, "tensor_core") <= limit
    x = _on_gpu(prefill_inputs([576], 96, 128, 128, "bf16", seed=23, s0_std=0.02))
    _check(x, *_both(x))
    assert K.kda_device_status() == 0
