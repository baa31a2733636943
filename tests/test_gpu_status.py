"""Failure detection without a GPU fault: a bounded device-side wait on a
barrier that nothing completes runs out, the kernel returns, the host reads
MOE_ERR_TIMEOUT, and the context stays usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    from group_limited_routed_moe_b200 import moe
    assert moe.get_device_status(0) == moe.MOE_OK
    moe.set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        moe.selftest_wait_timeout()
        torch.cuda.synchronize()
        assert moe.get_device_status(0) == moe.MOE_ERR_TIMEOUT
        assert "ran out" in moe.last_error()
        # status was cleared by the read; the context still runs kernels
        assert moe.get_device_status(0) == moe.MOE_OK
        a = torch.arange(10, device="cuda")
        assert int(a.sum()) == 45
    finally:
        moe.set_wait_timeout_ns(2_000_000_000)
