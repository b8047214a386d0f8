"""Failure detection without a GPU fault: the kernels' waits are bounded, and a
wait that runs out is reported through the device status word.

The self-test kernel waits on an mbarrier that nothing arrives on (the "flag
that nothing sets"); it must give up after its limit, the next status read
must return CIDER_ERR_TIMEOUT, and the context must stay usable: a linear run
right after gives the correct result and a clean status.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import act, check_y, dev, dev_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_reports_timeout_and_context_survives():
    cider.cider_device_status()  # start clean
    cider.cider_test_bounded_wait(20_000_000)  # 20 ms
    with pytest.raises(cider.CiderError) as e:
        cider.cider_device_status()
    assert e.value.status == 4  # CIDER_ERR_TIMEOUT
    cider.cider_device_status()  # cleared by the read above
    # the context is intact: a normal call still computes the right answer
    M, N, K = 130, 264, 512
    x = act(M, K, seed=3)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=3))
    y = cider.cider_w8a8_linear_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    check_y(y, oracle.linear_pc(x, qw, sw), oracle.F16)
    cider.cider_device_status()


def test_bounded_wait_limits_are_checked():
    with pytest.raises(cider.CiderError):
        cider.cider_test_bounded_wait(0)
    with pytest.raises(cider.CiderError):
        cider.cider_test_bounded_wait(10**9)
