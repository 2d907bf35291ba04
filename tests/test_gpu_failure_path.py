"""The failure path of the kernels' bounded waits, exercised without a GPU fault: a wait for
a barrier phase that nothing completes must give up after its limit, record W4_ERR_TIMEOUT
in the device status word, return, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import cuda, np_of

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_reports_timeout():
    assert w4.w4_device_status() == 0
    t0 = time.perf_counter()
    w4.w4_selftest_bounded_wait(20_000_000)  # 20 ms
    code = w4.w4_device_status()  # synchronizes
    dt = time.perf_counter() - t0
    assert code == 8, w4.STATUS.get(code, code)  # W4_ERR_TIMEOUT
    assert 0.015 <= dt < 5.0, dt
    # the status word was cleared by the read, and the context still runs kernels correctly
    assert w4.w4_device_status() == 0
    W = synth.normal((64, 256), 0.02, 0, 901)
    codes, scales, _, _ = w4.alloc_quantized(64, 256, 32, "sym", device=cuda(), chosen=False)
    w4.w4_quantize(W.to(cuda()), 64, 256, 32, "sym", [1.0], codes, scales, None, None)
    rc, rs, _, _ = oracle.quantize(synth.bf16_bits(W), 32, "sym", [1.0], want_chosen=False)
    assert np.array_equal(np_of(codes), rc)
    assert w4.w4_device_status() == 0


def test_bounded_wait_limit_is_validated():
    with pytest.raises(w4.W4Error):
        w4.w4_selftest_bounded_wait(10)
    with pytest.raises(w4.W4Error):
        w4.w4_selftest_bounded_wait(10 ** 10)
