"""Failure handling on the device, without a fault: the bounded mbarrier wait used by every
role of the prefill kernel runs in a small self-test kernel whose wait is made to run out
(a barrier phase nothing completes), is aborted by another thread, or completes. The
timeout must reach the host as GDN_ERR_TIMEOUT through the device error word, the other two
must leave no error, and the context must stay usable afterwards."""
import pytest
import torch

from tests.test_gpu_parity import check_prefill, custom

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def test_bounded_wait_times_out_and_reports():
    assert gdn.device_error() == "GDN_OK"
    assert gdn.selftest_bounded_wait(2_000_000, mode=0) == "GDN_ERR_TIMEOUT"
    assert gdn.device_error() == "GDN_OK"          # reading the status clears it


def test_bounded_wait_abort_and_completion_leave_no_error():
    assert gdn.selftest_bounded_wait(2_000_000, mode=1) == "GDN_OK"
    assert gdn.selftest_bounded_wait(2_000_000, mode=2) == "GDN_OK"


def test_context_usable_after_a_timeout():
    assert gdn.selftest_bounded_wait(1_000_000, mode=0) == "GDN_ERR_TIMEOUT"
    check_prefill(custom("bf16", (130, 64), 2, 128, 64, seed=17))
