"""The one-shot decode kernel (1 <= M <= 4, the automatic choice where its plan
fits) against the oracle.  One CTA of 1024 threads per SM owns a contiguous
range of weight rows and requests all of them at once by bulk copies of at
most 16 KB; its 32 warps take equal contiguous runs of 512-weight passes,
which may start and end inside a row, and each warp waits only for the
copies its passes lie in.  Shapes are chosen for the corners of that plan:

* the pages' decode shapes (per channel N = 10240, K = 2560: 70 rows of
  2.5 KB per CTA, 11 copies; per group N = 2560, K = 10240: 18 rows of 10 KB;
  W4A8 N = 12288, K = 4096);
* rows met by many warps (K = 16384: 32 passes per row, 32 slots), rows met
  by one warp, runs that end inside a row or inside a copy;
* a last pass of a row only partly filled (K = 528, 1040, 1088, 2576);
* fewer rows than SMs (N = 8, 16, 128, 136, 144: one row per CTA, most warps
  idle);
* shapes past the plan (a CTA's weight rows beyond shared memory, or more
  than two 16-byte chunks of x per thread), which take the register-ring
  kernel;
* all-zero tokens, both input dtypes, M = 1 .. 4.

Per channel the row sums are exact integers, so the one-shot and register-ring
kernels must agree bit for bit; per group the fp32 sums are added in a fixed
order, so repeated calls must agree bit for bit.  Parity bar as everywhere:
the row-relative fp16 (or bf16) tolerance."""
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
    cider.cider_test_set_small_m_kernel(4)
    yield
    cider.cider_test_set_small_m_kernel(0)
    cider.cider_set_small_m_threshold(old)
    cider.cider_device_status()


def _pc(M, N, K, seed, dt=F16):
    x = act(M, K, seed=seed, dt=dt)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=seed + 1))
    return x, qw, sw


PC_CASES = [(10240, 2560), (2056, 4096), (152, 528), (296, 1040), (144, 8192), (8, 16), (16, 512), (128, 256),
            (10240, 2576), (136, 32768), (144, 16384)]


@pytest.mark.parametrize("N,K", PC_CASES)
@pytest.mark.parametrize("M", [1, 2, 4])
def test_shot_pc(M, N, K):
    x, qw, sw = _pc(M, N, K, seed=M * 11 + N + K)
    y = cider.cider_w8a8_linear_pc(dev_bits(x, F16), dev(qw), dev(sw))
    check_y(y, oracle.linear_pc(x, qw, sw), F16)


PG_CASES = [(2560, 10240, 64), (2560, 10240, 128), (264, 32768, 64), (264, 16384, 64), (1032, 2560, 128),
            (296, 1088, 64), (8, 128, 64), (2056, 4096, 64)]


@pytest.mark.parametrize("N,K,gs", PG_CASES)
@pytest.mark.parametrize("M", [1, 3, 4])
def test_shot_pg(M, N, K, gs):
    x = act(M, K, seed=M * 5 + N + K + gs)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=N + K + gs), gs)
    y = cider.cider_w8a8_linear_pg(dev_bits(x, F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, oracle.linear_pg(x, qw, sw, gs), F16)


W4_CASES = [(12288, 4096, 64), (264, 2560, 128), (20480, 1024, 64), (2056, 4096, 64), (8, 64, 64)]


@pytest.mark.parametrize("N,K,gs", W4_CASES)
@pytest.mark.parametrize("M", [1, 4])
def test_shot_w4(M, N, K, gs):
    x = act(M, K, seed=M * 3 + N + K + gs)
    packed, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, seed=N + 2 * K + gs), gs)
    y = cider.cider_w4a8_linear_pg(dev_bits(x, F16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
    check_y(y, oracle.w4a8_linear_pg(x, packed, sw, gs), F16)


@pytest.mark.parametrize("mode", ["pc", "pg", "w4"])
def test_shot_bf16_and_zero_token(mode):
    M, N, K, gs = 4, 1032, 2560, 64
    x = act(M, K, seed=17, dt=BF16)
    x[2] = 0
    W = synth.weights(N, K, seed=18)
    if mode == "pc":
        qw, sw = oracle.quantize_weight_pc(W)
        y = cider.cider_w8a8_linear_pc(dev_bits(x, BF16), dev(qw), dev(sw))
        ref = oracle.linear_pc(x, qw, sw, xdt=BF16, ydt=BF16)
    elif mode == "pg":
        qw, sw = oracle.quantize_weight_pg(W, gs)
        y = cider.cider_w8a8_linear_pg(dev_bits(x, BF16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
        ref = oracle.linear_pg(x, qw, sw, gs, xdt=BF16, ydt=BF16)
    else:
        packed, sw = oracle.quantize_weight_int4_pg(W, gs)
        y = cider.cider_w4a8_linear_pg(dev_bits(x, BF16), dev(packed), dev(np.ascontiguousarray(sw.T)), gs)
        ref = oracle.w4a8_linear_pg(x, packed, sw, gs, xdt=BF16, ydt=BF16)
    check_y(y, ref, BF16)
    assert not y[2].any()


@pytest.mark.parametrize("M,N,K", [(1, 10240, 2560), (4, 2056, 4096), (3, 144, 8192), (2, 152, 528)])
def test_shot_pc_equals_register_ring(M, N, K):
    """Per channel both kernels add exact INT32 products and dequantize with the
    same expression: the outputs must be identical."""
    x, qw, sw = _pc(M, N, K, seed=M + N)
    xd, w, s = dev_bits(x, F16), dev(qw), dev(sw)
    y_shot = cider.cider_w8a8_linear_pc(xd, w, s)
    cider.cider_test_set_small_m_kernel(1)
    try:
        y_ring = cider.cider_w8a8_linear_pc(xd, w, s)
    finally:
        cider.cider_test_set_small_m_kernel(4)
    torch.cuda.synchronize()
    assert torch.equal(y_shot.view(torch.int16), y_ring.view(torch.int16))


@pytest.mark.parametrize("N,K,gs", [(2560, 10240, 64), (264, 16384, 64)])
def test_shot_pg_repeated_calls_agree(N, K, gs):
    """A row's pieces are added in warp order: the same call twice gives the same bits."""
    x = dev_bits(act(1, K, seed=3), F16)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=4), gs)
    w, s = dev(qw), dev(np.ascontiguousarray(sw.T))
    a = cider.cider_w8a8_linear_pg(x, w, s, gs)
    b = cider.cider_w8a8_linear_pg(x, w, s, gs)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shot_many_calls_in_a_row():
    """200 calls back to back on one stream (launches overlap through
    programmatic serialisation): the last outputs are still right."""
    M, N, K = 1, 2056, 4096
    xs = [act(M, K, seed=40 + i) for i in range(3)]
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=41))
    xd = [dev_bits(x, F16) for x in xs]
    w, s = dev(qw), dev(sw)
    ys = [cider.cider_w8a8_linear_pc(xd[i % 3], w, s) for i in range(200)]
    torch.cuda.synchronize()
    for i in (197, 198, 199):
        check_y(ys[i], oracle.linear_pc(xs[i % 3], qw, sw), F16)
