"""The device-side timeout path on a GPU, without a fault: one kernel waits,
with the conv kernels' bounded wait, on an mbarrier that nothing arrives at.
The wait gives up after its limit, sets its bit in the device error word and
the kernel returns; mqv_device_errors reports MQV_ERR_TIMEOUT with that bit
and clears it, and the context keeps working."""
import ctypes

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv

pytestmark = pytest.mark.gpu

MQV_ERR_TIMEOUT = 5
SELFTEST_BIT = 8


def test_bounded_wait_gives_up_and_reports():
    assert mqv.device_errors() == 0                         # start clean
    limit = 4_000_000                                       # about 2 ms at 1.9-2 GHz
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    mqv.selftest_wait_timeout(limit)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    flags = ctypes.c_uint32()
    st = mqv.lib().mqv_device_errors(ctypes.byref(flags), None)
    assert st == MQV_ERR_TIMEOUT and flags.value == SELFTEST_BIT
    assert b"timed out" in mqv.lib().mqv_last_error()
    # the wait lasted its limit (SM clocks stay below 2.1 GHz) and no longer
    assert limit / 2.1e6 <= ms < 1000.0, ms
    # read once, the word is clear, and the context still runs kernels
    assert mqv.device_errors() == 0
    x = torch.randn(64 * 64, device="cuda")
    q = mqv.quantize(x, 64, 64, "nvfp4")
    torch.cuda.synchronize()
    assert mqv.device_errors() == 0
    assert np.isfinite(mqv.dequantize(q).cpu().numpy()).all()


def test_timeout_flag_accumulates_across_calls_until_read():
    mqv.device_errors()
    mqv.selftest_wait_timeout(100_000)
    mqv.selftest_wait_timeout(100_000)
    assert mqv.device_errors() == SELFTEST_BIT
    assert mqv.device_errors() == 0
