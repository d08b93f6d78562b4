"""The bounded-wait watchdog, exercised without faulting or hanging the GPU:
a kernel waits on an mbarrier that nothing arrives on, gives up after a short
cycle budget, and the host reads FA_ERR_TIMEOUT from the status word."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_then_cleared():
    from flashattention_attention_b200 import fa
    assert fa.check_device_error() == fa.FA_OK
    assert fa.selftest_watchdog(200_000) == fa.FA_OK
    assert fa.check_device_error() == fa.FA_ERR_TIMEOUT
    assert fa.check_device_error() == fa.FA_OK  # the word is cleared after reading
    # the context stays usable
    x = torch.ones(4, 64, device="cuda")
    codes, scales = fa.compress_kv(x)
    torch.cuda.synchronize()
    assert int(codes.sum()) == 4 * 64 * 127
