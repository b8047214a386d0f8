"""The W8A16 decode kernels (no activation quantization; Cider README, section
"Metal Kernel 流水线", Decode: the per-channel and the per-group INT8 MV
kernels) against the oracle's W8A16 modes, within the row-relative
tolerance, for 1 <= M <= 4, both input dtypes and both output dtypes,
including shapes whose K is split across warps, whose rows wrap the ring of
shared-memory stages, the one-shot kernel's corners (forced against the
register ring), and the argument checks."""
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


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(10240, 2560), (2560, 10240), (264, 1040), (8, 16)])
def test_w8a16_mv(kernel, M, N, K):
    """The automatic choice (the register ring per channel) and the ring
    forced, on the same shapes; the one-shot form is forced in the tests
    below."""
    x = act(M, K, seed=M + N + K)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=N + K))
    cider.cider_test_set_small_m_kernel(kernel)
    try:
        y = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    finally:
        cider.cider_test_set_small_m_kernel(0)
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


# ---- per-group weight scales (cider_w8a16_mv_pg) ---------------------------------

@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("N,K,gs", [(2560, 10240, 64), (2560, 10240, 128), (10240, 2560, 64), (264, 1088, 64),
                                    (20480, 1024, 128), (8, 64, 64), (136, 32768, 128), (136, 16384, 128)])
def test_w8a16_mv_pg(M, N, K, gs):
    x = act(M, K, seed=M + N + K + gs)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=N + K + gs), gs)
    args = (dev_bits(x, oracle.F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
    if M * ((K // 16 + 31) // 32) * 2048 > 160 * 1024:  # staged fp32 rows beyond shared memory
        with pytest.raises(cider.CiderError, match="shared memory"):
            cider.cider_w8a16_mv_pg(*args)
        return
    y = cider.cider_w8a16_mv_pg(*args)
    check_y(y, oracle.w8a16_linear_pg(x, qw, sw, gs), oracle.F16)


@pytest.mark.parametrize("xdt,ydt", [(oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16)])
def test_w8a16_mv_pg_dtypes_and_zero_token(xdt, ydt):
    M, N, K, gs = 3, 1032, 4096, 64
    x = act(M, K, seed=19, dt=xdt)
    x[2] = 0
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=20), gs)
    out = torch.bfloat16 if ydt == oracle.BF16 else torch.float16
    y = cider.cider_w8a16_mv_pg(dev_bits(x, xdt), dev(qw), dev(np.ascontiguousarray(sw.T)), gs, out_dtype=out)
    check_y(y, oracle.w8a16_linear_pg(x, qw, sw, gs, xdt=xdt, ydt=ydt), ydt)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y[2]).item() == 0


def test_w8a16_mv_pg_one_group_equals_per_channel_kernel_shape():
    """With gs = 128 = K the per-group product is the per-channel one; both
    kernels must agree with the oracle on the same inputs."""
    M, N, K = 2, 264, 128
    x = act(M, K, seed=21)
    qw, sw = oracle.quantize_weight_pc(synth.weights(N, K, seed=22))
    y_pg = cider.cider_w8a16_mv_pg(dev_bits(x, oracle.F16), dev(qw), dev(sw[None, :].copy()), 128)
    y_pc = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
    ref = oracle.w8a16_linear_pc(x, qw, sw)
    check_y(y_pg, ref, oracle.F16)
    check_y(y_pc, ref, oracle.F16)


def test_w8a16_mv_pg_argument_checks():
    N, K = 264, 1024
    x = dev_bits(act(1, K, seed=1), oracle.F16)
    w = dev(np.zeros((N, K), np.int8))
    with pytest.raises(cider.CiderError):  # gs must be 64 or 128
        cider.cider_w8a16_mv_pg(x, w, dev(np.ones((K // 32, N), np.float32)), 32)
    with pytest.raises(cider.CiderError):  # decode shapes only
        cider.cider_w8a16_mv_pg(dev_bits(act(5, K, seed=1), oracle.F16), w, dev(np.ones((K // 64, N), np.float32)), 64)
    with pytest.raises(cider.CiderError):  # staged rows beyond shared memory
        cider.cider_w8a16_mv_pg(dev_bits(act(4, 16384, seed=1), oracle.F16), dev(np.zeros((8, 16384), np.int8)),
                                dev(np.ones((256, 8), np.float32)), 64)


@pytest.mark.parametrize("kernel", [2, 3])
def test_w8a16_mv_bulk_kernel(kernel):
    """The bulk-staged W8A16 kernels (selectable by the test switch) on the
    per-channel and per-group forms."""
    M, N, K, gs = 2, 2056, 4096, 64
    x = act(M, K, seed=kernel)
    W = synth.weights(N, K, seed=kernel + 1)
    qc, sc = oracle.quantize_weight_pc(W)
    qg, sg = oracle.quantize_weight_pg(W, gs)
    cider.cider_test_set_small_m_kernel(kernel)
    try:
        y_pc = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qc), dev(sc))
        y_pg = cider.cider_w8a16_mv_pg(dev_bits(x, oracle.F16), dev(qg), dev(np.ascontiguousarray(sg.T)), gs)
    finally:
        cider.cider_test_set_small_m_kernel(0)
    check_y(y_pc, oracle.w8a16_linear_pc(x, qc, sc), oracle.F16)
    check_y(y_pg, oracle.w8a16_linear_pg(x, qg, sg, gs), oracle.F16)


# ---- the one-shot kernel (A16 mode) against the register ring -----------------

@pytest.mark.parametrize("kernel", [1, 4])
@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("mode,N,K,gs", [("pc", 10240, 2560, 0), ("pg", 2560, 10240, 64), ("pg", 2560, 10240, 128),
                                         ("pc", 144, 16384, 0), ("pg", 264, 16384, 128), ("pc", 152, 1040, 0),
                                         ("pg", 296, 1088, 64), ("pg", 8, 128, 64)])
def test_w8a16_one_shot_and_register_ring(kernel, M, mode, N, K, gs):
    """Both W8A16 kernels on the one-shot kernel's corners: the decode shapes,
    rows met by many warps (K = 16384), partial last passes (K = 1040, 1088)
    and fewer rows than SMs."""
    if K == 16384 and M > 1:
        pytest.skip("M x K beyond the staged activations of the register-ring kernel")
    x = act(M, K, seed=M + N + K + gs + kernel)
    W = synth.weights(N, K, seed=N + K + gs)
    cider.cider_test_set_small_m_kernel(kernel)
    try:
        if mode == "pc":
            qw, sw = oracle.quantize_weight_pc(W)
            y = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.F16), dev(qw), dev(sw))
            ref = oracle.w8a16_linear_pc(x, qw, sw)
        else:
            qw, sw = oracle.quantize_weight_pg(W, gs)
            y = cider.cider_w8a16_mv_pg(dev_bits(x, oracle.F16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs)
            ref = oracle.w8a16_linear_pg(x, qw, sw, gs)
    finally:
        cider.cider_test_set_small_m_kernel(0)
    check_y(y, ref, oracle.F16)


@pytest.mark.parametrize("mode", ["pc", "pg"])
def test_w8a16_one_shot_bf16(mode):
    M, N, K, gs = 2, 2056, 4096, 64
    x = act(M, K, seed=5, dt=oracle.BF16)
    x[1] = 0
    W = synth.weights(N, K, seed=6)
    if mode == "pc":
        qw, sw = oracle.quantize_weight_pc(W)
        y = cider.cider_w8a16_mv_pc(dev_bits(x, oracle.BF16), dev(qw), dev(sw), out_dtype=torch.bfloat16)
        ref = oracle.w8a16_linear_pc(x, qw, sw, xdt=oracle.BF16, ydt=oracle.BF16)
    else:
        qw, sw = oracle.quantize_weight_pg(W, gs)
        y = cider.cider_w8a16_mv_pg(dev_bits(x, oracle.BF16), dev(qw), dev(np.ascontiguousarray(sw.T)), gs,
                                    out_dtype=torch.bfloat16)
        ref = oracle.w8a16_linear_pg(x, qw, sw, gs, xdt=oracle.BF16, ydt=oracle.BF16)
    check_y(y, ref, oracle.BF16)
    assert not y[1].any()
