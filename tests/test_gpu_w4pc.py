"""W4A8 with one scale per output channel (Cider README, table "量化": INT4
weights, zero point 8, per column) against the oracle: the INT4 packer bit
for bit, the linear within the row-relative tolerance on ragged shapes, both
input dtypes, forced split-K and sampled rows of the full 2048 x 12288 x 4096
shape."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import act, check_y, dev, dev_bits

pytestmark = pytest.mark.gpu
F16, BF16 = oracle.F16, oracle.BF16

SHAPES = [(1, 256, 1024), (3, 136, 2560), (16, 128, 256), (129, 264, 1280), (300, 520, 2560), (130, 264, 192),
          (64, 512, 4096)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_device_status()


@pytest.mark.parametrize("N,K", [(12288, 4096), (5, 34), (1, 2), (264, 1280)])
def test_pack_weight_int4_pc_bit_exact(N, K):
    W = np.random.default_rng(N + K).standard_t(3, size=(N, K)).astype(np.float32) * 0.02
    W[0, : min(K, 7)] = 0.0
    p, s = cider.cider_pack_weight_int4_pc(dev(W))
    po, so = oracle.quantize_weight_int4_pc(W)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(p.cpu().numpy(), po)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("xdt", [F16, BF16])
def test_w4a8_linear_pc(M, N, K, xdt):
    x = act(M, K, seed=5 * M + N + K, dt=xdt)
    packed, sw = oracle.quantize_weight_int4_pc(synth.weights(N, K, seed=3 * N + K))
    y = cider.cider_w4a8_linear_pc(dev_bits(x, xdt), dev(packed), dev(sw))
    check_y(y, oracle.w4a8_linear_pc(x, packed, sw, xdt=xdt, ydt=xdt), xdt)


def test_w4a8_linear_pc_full_shape_sampled_rows():
    M, N, K = 2048, 12288, 4096
    x = act(M, K, seed=11)
    packed, sw = oracle.quantize_weight_int4_pc(synth.weights(N, K, seed=12))
    y = cider.cider_w4a8_linear_pc(dev_bits(x, F16), dev(packed), dev(sw))
    rows = np.array([0, 1, 777, 1500, 2047])
    check_y(y[torch.from_numpy(rows).cuda()], oracle.w4a8_linear_pc(x[rows], packed, sw), F16)


@pytest.mark.parametrize("pieces", [2, 3, 7])
def test_w4a8_linear_pc_forced_split(pieces):
    M, N, K = 200, 264, 2560
    x = act(M, K, seed=pieces)
    packed, sw = oracle.quantize_weight_int4_pc(synth.weights(N, K, seed=pieces + 1))
    cider.cider_test_set_split_k(pieces)
    try:
        y = cider.cider_w4a8_linear_pc(dev_bits(x, F16), dev(packed), dev(sw))
    finally:
        cider.cider_test_set_split_k(0)
    check_y(y, oracle.w4a8_linear_pc(x, packed, sw), F16)


def test_w4a8_gemm_pc_q_matches_linear():
    M, N, K = 200, 264, 1024
    x = act(M, K, seed=2)
    xd = dev_bits(x, F16)
    packed, sw = oracle.quantize_weight_int4_pc(synth.weights(N, K, seed=2))
    cider.cider_test_set_split_k(1)
    try:
        q, s = cider.cider_quantize_act(xd)
        torch.testing.assert_close(cider.cider_w4a8_gemm_pc_q(q, s, dev(packed), dev(sw)),
                                   cider.cider_w4a8_linear_pc(xd, dev(packed), dev(sw)), rtol=0, atol=0)
    finally:
        cider.cider_test_set_split_k(0)


def test_w4a8_linear_pc_argument_checks():
    x = dev_bits(act(4, 48, seed=1), F16)
    with pytest.raises(cider.CiderError):  # K % 32
        cider.cider_w4a8_linear_pc(x, dev(np.zeros((8, 24), np.uint8)), dev(np.ones(8, np.float32)))
    with pytest.raises(cider.CiderError):  # odd K for the packer
        cider.cider_pack_weight_int4_pc(dev(np.ones((2, 3), np.float32)))
