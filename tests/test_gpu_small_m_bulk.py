"""The bulk-staged decode kernel (1 <= M <= 4; selected by the test switch --
the register-ring kernel, which measured faster, is the default) against the
oracle, on shapes chosen for the corners of its plan (one CTA per SM owns a
contiguous range of weight rows and streams it through a ring of
shared-memory stages of R rows, eight warps as R rows x 8/R K-slices):

* more stages per CTA than ring slots, so slots are reused (N = 20480);
* a CTA's last stage only partly filled (rows per CTA not a multiple of R);
* K-slices (R < 8 at K = 10240) and a slice whose lanes do not all have a
  chunk (K = 2576: 161 chunks);
* the smallest row (K = 16, one chunk) and the largest (K = 32768, R = 1);
* fewer rows than SMs (N = 8: a one-CTA grid);
* a plan that does not fit in shared memory (per group, K = 32768, M = 4),
  which takes the register-ring kernel instead;
* all-zero tokens, both input dtypes, per channel, per group and W4A8.

Parity bar as everywhere: the row-relative fp16 (or bf16) tolerance."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from w8a8_activation_quantized_b200 import synth
from tests.parity import act, check_y, dev, dev_bits

pytestmark = pytest.mark.gpu
F16, BF16 = oracle.F16, oracle.BF16


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    old = cider.cider_get_small_m_threshold()
    cider.cider_set_small_m_threshold(4)
    cider.cider_test_set_small_m_kernel(2)
    yield
    cider.cider_test_set_small_m_kernel(0)
    cider.cider_set_small_m_threshold(old)
    cider.cider_device_status()


PC_CASES = [(20480, 2560), (10240, 2560), (264, 2576), (8, 16), (136, 32768), (2560, 10240), (1032, 4096)]


@pytest.mark.parametrize("N,K", PC_CASES)
@pytest.mark.parametrize("M", [1, 2, 4])
def test_small_m_pc(M, N, K):
    x = act(M, K, seed=M * 7 + N + K)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=N + K))
    y = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    check_y(y, oracle.linear_pc(x, qw, sw), F16)


PG_CASES = [(2560, 10240, 64), (2560, 10240, 128), (20480, 1280, 64), (264, 32768, 64), (8, 128, 64),
            (1032, 2560, 128)]


@pytest.mark.parametrize("N,K,gs", PG_CASES)
@pytest.mark.parametrize("M", [1, 3, 4])
def test_small_m_pg(M, N, K, gs):
    x = act(M, K, seed=M * 5 + N + K + gs)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=N + K + gs), gs)
    y = cider.cider_w8a8_linear_pg(dev_bits(x, F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, oracle.linear_pg(x, qw, sw, gs), F16)


W4_CASES = [(12288, 4096, 64), (264, 2560, 128), (20480, 1024, 64), (8, 64, 64)]


@pytest.mark.parametrize("N,K,gs", W4_CASES)
@pytest.mark.parametrize("M", [1, 4])
def test_small_m_w4(M, N, K, gs):
    x = act(M, K, seed=M * 3 + N + K + gs)
    packed, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, seed=N + 2 * K + gs), gs)
    y = cider.cider_w4a8_linear_pg(dev_bits(x, F16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, oracle.w4a8_linear_pg(x, packed, sw, gs), F16)


@pytest.mark.parametrize("mode", ["pc", "pg"])
def test_small_m_bf16_and_zero_token(mode):
    M, N, K, gs = 4, 1032, 2560, 64
    x = act(M, K, seed=17, dt=BF16)
    x[1] = 0
    W = synth.weights(N, K, seed=18)
    if mode == "pc":
        qw, sw = oracle.quantize_weight_pc(W)
        y = cider.cider_w8a8_linear_pc(dev_bits(x, BF16), dev(qw), dev(sw))
        ref = oracle.linear_pc(x, qw, sw, xdt=BF16, ydt=BF16)
    else:
        qw, sw = oracle.quantize_weight_pg(W, gs)
        y = cider.cider_w8a8_linear_pg(dev_bits(x, BF16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
        ref = oracle.linear_pg(x, qw, sw, gs, xdt=BF16, ydt=BF16)
    check_y(y, ref, BF16)
    assert not y[1].any()


def test_small_m_repeated_calls_agree():
    """The same call twice in a row on one stream gives identical bits (the
    slices are added in a fixed order; nothing carries over between calls)."""
    M, N, K, gs = 1, 2560, 10240, 64
    x = dev_bits(act(M, K, seed=3), F16)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=4), gs)
    w, s = dev(qw), dev(np.ascontiguousarray(sw.T))
    a = cider.cider_w8a8_linear_pg(x, w, s, gs)
    b = cider.cider_w8a8_linear_pg(x, w, s, gs)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("mode", ["pc", "pg", "w4"])
def test_small_m_each_kernel(kernel, mode):
    """The test switch's three decode kernels (register ring, bulk-staged with
    the whole shared memory, bulk-staged within half of it) on one shape."""
    M, N, K, gs = 2, 2056, 4096, 64
    x = act(M, K, seed=kernel * 10 + len(mode))
    W = synth.weights(N, K, seed=77)
    cider.cider_test_set_small_m_kernel(kernel)
    try:
        if mode == "pc":
            qw, sw = oracle.quantize_weight_pc(W)
            y = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
            ref = oracle.linear_pc(x, qw, sw)
        elif mode == "pg":
            qw, sw = oracle.quantize_weight_pg(W, gs)
            y = cider.cider_w8a8_linear_pg(dev_bits(x, F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
            ref = oracle.linear_pg(x, qw, sw, gs)
        else:
            packed, sw = oracle.quantize_weight_int4_pg(W, gs)
            y = cider.cider_w4a8_linear_pg(dev_bits(x, F16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
            ref = oracle.w4a8_linear_pg(x, packed, sw, gs)
    finally:
        cider.cider_test_set_small_m_kernel(2)  # this module's setting
    check_y(y, ref, F16)


@pytest.mark.parametrize("M,K", [(12, 4096), (3, 16384), (16, 3072)])
def test_register_ring_at_48k_of_codes(M, K):
    """The register-ring kernel stages M x K codes in shared memory; at exactly
    48 KB (plus its static shared memory) the launch must opt in to more than
    the default, or it is refused."""
    N = 264
    x = act(M, K, seed=M + K)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=K))
    old = cider.cider_get_small_m_threshold()
    cider.cider_set_small_m_threshold(16)
    cider.cider_test_set_small_m_kernel(1)
    try:
        y = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    finally:
        cider.cider_test_set_small_m_kernel(2)  # this module's setting
        cider.cider_set_small_m_threshold(old)
    check_y(y, oracle.linear_pc(x, qw, sw), F16)
