"""Failure detection without a GPU fault: a wait whose producer never arrives
ends in a status code after its time budget, and the context stays usable."""
import pytest
import torch

from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import make_inputs
from gpu_helpers import run_fwd_bwd

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    s = torch.cuda.current_stream(0)
    assert ga.gptattn_get_device_status(s) == ga.GPTATTN_OK
    assert ga.gptattn_selftest_wait_timeout(2_000_000, s) == ga.GPTATTN_OK   # 2 ms budget
    assert ga.gptattn_get_device_status(s) == ga.GPTATTN_ERR_TIMEOUT
    assert ga.gptattn_get_device_status(s) == ga.GPTATTN_OK                   # read clears it
    qkv, dy = make_inputs(1, 130, 2, 64, dtype=torch.bfloat16, seed=1)
    y, lse, dqkv = run_fwd_bwd(qkv, dy, 2)                                    # still works
    assert (abs(y) < 100).all()


def test_invalid_call_enqueues_nothing():
    s = torch.cuda.current_stream(0)
    before = ga.gptattn_launch_count()
    x = torch.zeros(8, device="cuda")
    assert ga.gptattn_fwd(x, x, x, 1, 4, 96, 3, ga.GPTATTN_BF16, s) == ga.GPTATTN_ERR_UNSUPPORTED
    assert ga.gptattn_launch_count() == before
