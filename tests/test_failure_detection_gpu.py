"""Failure detection on the GPU without a fault (B200 only).

A kernel whose mbarrier wait is never satisfied gives up after its limit,
records KDA_ERR_TIMEOUT in the library's device status word and returns; the
host reads the status, the word is cleared by the read, and the context stays
usable -- a prefill afterwards still matches the oracle.
"""
import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as K
from linear_attention_serving_prefill_b200.workloads import prefill_inputs
from oracle import oracle
from tests.kda_testutil import TOL_BF16, relerr, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert K.kda_device_status() == 0
    K.kda_selftest_wait_timeout(50_000_000)          # 50 ms
    assert K.kda_device_status() == 5                # KDA_ERR_TIMEOUT
    assert K.kda_device_status() == 0                # cleared by the read
    x = prefill_inputs([70, 3], 2, 128, 128, "bf16", seed=31, s0_std=0.02)
    xd = {key: (val.cuda() if isinstance(val, torch.Tensor) and key != "cu_seqlens_host" else val)
          for key, val in x.items()}
    o, S = K.kda_prefill(xd["q"], xd["k"], xd["v"], xd["z"], xd["A"], xd["beta"], xd["cu_seqlens"],
                         x["cu_seqlens_host"], initial_state=xd["initial_state"])
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.prefill(x["q"], x["k"], x["v"], x["z"], x["A"], x["beta"],
                                  x["cu_seqlens_host"], x["initial_state"])
    assert relerr(to_np(o), ref_o) <= TOL_BF16
    assert relerr(to_np(S), ref_S) <= TOL_BF16
    assert K.kda_device_status() == 0
