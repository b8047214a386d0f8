"""The W8A16 decode kernel (no activation quantization; Cider README, section
"Metal Kernel 流水线", Decode) against the oracle's W8A16 mode, within the
row-relative tolerance, for 1 <= M <= 4, both input dtypes and both output
dtypes, including shapes whose K is split across warps."""
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
    yield
    cider.cider_device_status()


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(10240, 2560), (2560, 10240), (264, 1040), (8, 16)])
def test_w8a16_mv(M, N, K):
    x = act(M, K, seed=M + N + K)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=N + K))
    y = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    check_y(y, oracle.w8a16_linear_pc(x, qw, sw), oracle.F16)


@pytest.mark.parametrize("xdt,ydt", [(oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16), (oracle.BF16, oracle.F16)])
def test_w8a16_mv_dtypes(xdt, ydt):
    M, N, K = 2, 1032, 4096
    x = act(M, K, seed=9, dt=xdt)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=10))
    out = torch.bfloat16 if ydt == oracle.BF16 else torch.float16
    y = cider.cider_w8a16_mv_pc(dev_bits(x, xdt), dev(qw), dev(sw), out_dtype=out)
    check_y(y, oracle.w8a16_linear_pc(x, qw, sw, xdt=xdt, ydt=ydt), ydt)


def test_w8a16_mv_zero_token_and_argument_checks():
    N, K = 264, 1024
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=3))
    x = act(2, K, seed=3)
    x[1] = 0
    y = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    torch.cuda.synchronize()
    assert torch.count_nonzero(y[1]).item() == 0
    check_y(y, oracle.w8a16_linear_pc(x, qw, sw), oracle.F16)
    with pytest.raises(cider.CiderError):  # decode shapes only
        cider.cider_w8a16_mv_pc(dev_bits(act(5, K, seed=1), oracle.F16), dev(qw), dev(sw))
    with pytest.raises(cider.CiderError):  # activation rows must fit in shared memory
        cider.cider_w8a16_mv_pc(dev_bits(act(4, 16384, seed=1), oracle.F16),
                                dev(np.zeros((8, 16384), np.int8)), dev(np.ones(8, np.float32)))
