"""Failure detection on the GPU without a fault: a wait that nothing completes runs out after
its time limit, the kernel returns, and the host reads the status and the wait's site."""
import time

import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api

pytestmark = [pytest.mark.gpu, pytest.mark.status_checked]


def test_bounded_wait_times_out_and_reports():
    assert api.check_status() == 0
    api.timeout_site()                                     # clear any stale record
    t0 = time.time()
    api.selftest_wait_timeout()
    assert api.check_status() == 4                         # QK4V8_ERR_TIMEOUT
    dt = time.time() - t0
    assert 0.9 < dt < 10.0
    site = api.timeout_site()
    assert site is not None and site["kernel"] == "selftest"
    assert api.timeout_site() is None                      # cleared by the read
    assert api.check_status() == 0                         # status cleared too
    # the context is still usable
    x = torch.randn(64, 128, device="cuda", dtype=torch.bfloat16)
    q = api.quantize_nvfp4(x)
    assert api.check_status() == 0 and q.codes.shape == (64, 64)
