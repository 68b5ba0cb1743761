"""Failure detection without a GPU fault: a wait that nothing completes gives
up after its limit (about 10 ms here), the kernel records a timeout in the
workspace status word and returns, and the context stays usable."""
import pytest
import torch

import serving_block_union_b200 as ca

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok):
    ws = ca.new_workspace(1, 4, 1, 64, 64)
    ca.selftest_bounded_wait(ws, limit_cycles=20_000_000)
    assert ca.read_device_status(ws) == ca.CA_ERR_TIMEOUT
    # the context still runs work afterwards
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
    ws2 = ca.new_workspace(1, 4, 1, 64, 64)
    assert ca.read_device_status(ws2) == ca.CA_OK


def test_selftest_rejects_bad_limits(cuda_ok):
    ws = ca.new_workspace(1, 4, 1, 64, 64)
    with pytest.raises(ca.CAError):
        ca.selftest_bounded_wait(ws, limit_cycles=0)
