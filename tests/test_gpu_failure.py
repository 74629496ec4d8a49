"""The library's failure path on the GPU without a fault: a wait that runs out of time returns
an error status the host reads, and the context stays usable."""
import time

import pytest
import torch

import verify_step_b200 as sd
from tests.gpu_util import DEV, status_ok

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    sd.sd_device_status_clear()
    torch.cuda.synchronize()
    t = time.perf_counter()
    sd.sd_selftest_bounded_wait()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t
    assert sd.sd_device_status_read() == sd.SD_ERR_TIMEOUT
    assert 1.5 < elapsed < 30.0  # the 2 s limit, not a hang
    sd.sd_device_status_clear()
    # the context still runs work afterwards
    x = torch.arange(1 << 20, device=DEV, dtype=torch.float32)
    assert float(x.sum().item()) == pytest.approx((1 << 20) * ((1 << 20) - 1) / 2)
    assert status_ok()
