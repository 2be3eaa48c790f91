"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies runs out, the kernel returns, the host reads the timeout status,
and the context keeps working."""
import pytest
import torch

import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import small_case

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    w4.w4a8_check_device_error()                      # latch starts clear
    w4.w4a8_selftest_wait_timeout(0.05)
    with pytest.raises(w4.W4A8Error) as ei:
        w4.w4a8_check_device_error()
    assert "DEVICE_TIMEOUT" in str(ei.value)
    w4.w4a8_check_device_error()                      # reading it cleared it
    # the context is still usable: a forward runs and gives the same bits twice
    cfg = workloads.CONFIGS[0]
    hidden, logits, w13, w2 = small_case(cfg)
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    a = layer(hidden.cuda(), logits.cuda())
    b = layer(hidden.cuda(), logits.cuda())
    w4.w4a8_check_device_error()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_selftest_rejects_bad_timeout():
    with pytest.raises(w4.W4A8Error):
        w4.w4a8_selftest_wait_timeout(0.0)
    with pytest.raises(w4.W4A8Error):
        w4.w4a8_selftest_wait_timeout(11.0)
