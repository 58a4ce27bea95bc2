"""Failure detection without a GPU fault (GPU): a kernel waiting on an
mbarrier that nobody arrives on gives up after its iteration limit, records
DD_ERR_TIMEOUT in the device error word and returns; the context stays usable."""
import pytest
import torch

from speculative_verification_cover_b200 import dd

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert dd.dd_get_device_error() == dd.DD_OK
    dd.dd_selftest_bounded_wait(1000)
    assert dd.dd_get_device_error() == dd.DD_ERR_TIMEOUT
    # cleared on read
    assert dd.dd_get_device_error() == dd.DD_OK
    # the context still works: a real call succeeds afterwards
    lt = torch.randn(1, 2, 512, device="cuda")
    stats = dd.RowStats.empty(1, 2)
    dd.dd_verify_logits(lt, lt.clone(), stats)
    torch.cuda.synchronize()
    assert torch.equal(stats.argmax_t[0].long(), lt[0].argmax(-1))
    assert dd.dd_get_device_error() == dd.DD_OK


def test_spin_limit_setting_round_trips():
    old = dd.dd_set_spin_limit(12345)
    assert dd.dd_set_spin_limit(old) == 12345
