"""Bounded device waits end with a status code, never a hang or a fault.

The diagnostic kernel waits, with the library's bounded wait, on a shared-memory barrier that
nothing completes (no trap, no bad address, no endless loop): after about a second the wait
gives up, the status word records the timeout, and the context keeps working.
"""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda):
    import cnn_convolution_nhwc_b200 as cb
    assert cb.conv_device_status(reset=True) == cb.CONV_OK
    t0 = time.time()
    assert cb.conv_selftest_wait_timeout() == cb.CONV_OK
    assert cb.conv_device_status(reset=True) == cb.CONV_ERR_DEVICE_TIMEOUT
    elapsed = time.time() - t0
    assert 0.2 < elapsed < 30, elapsed
    assert cb.conv_device_status() == cb.CONV_OK          # the reset cleared it
    # the context is intact: a convolution still runs and is right
    x = torch.ones((1, 1, 5, 5), device="cuda")
    w = torch.ones((1, 3, 3), device="cuda")
    y = cb.depthwise_fwd(x, w, None, pad=1)
    assert y[0, 0, 2, 2].item() == 9.0 and y[0, 0, 0, 0].item() == 4.0
    assert cb.conv_device_status() == cb.CONV_OK
