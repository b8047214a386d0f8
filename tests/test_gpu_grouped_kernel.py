"""The per-group GEMM kernel against the oracle on ragged shapes and at the
edge of its arithmetic: every group's TMEM buffer is first overwritten by a
kind::f16 MMA of constant operands (the bias 1.5 * 2^23) and the group's
kind::i8 MMAs accumulate onto it, so bit-exact INT32 per-group partials check
the bias and the accumulation together; the W8A8 per-group and W4A8 linears
are checked within the row-relative tolerance."""
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


def _gmajor(sw):
    """Oracle weight scales [N][G] -> the device layout [G][N]."""
    return dev(np.ascontiguousarray(sw.T))


def _codes(M, N, K, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int64).astype(np.int8)
    w = rng.integers(-128, 128, size=(N, K), dtype=np.int64).astype(np.int8)
    return q, w


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(256, 128, 128), (1, 8, 128), (257, 264, 384), (300, 520, 640),
                                   (130, 1160, 256), (513, 136, 1024)])
def test_gemm_i32_grouped_ragged(M, N, K, gs):
    q, w = _codes(M, N, K, seed=5 * M + N + K + gs)
    acc_g = cider.cider_test_gemm_i32_grouped(dev(q), dev(w), gs)
    np.testing.assert_array_equal(acc_g.cpu().numpy(), oracle.gemm_i32_grouped(q, w, gs))


def test_gemm_i32_grouped_extremes():
    """Products of magnitude 127 * 128 throughout: |partial| = gs * 16256 at
    gs = 128, the largest a group can reach with symmetric activation codes,
    still inside the +-2^22 window the float view of the bias allows."""
    M, N, K, gs = 260, 136, 384, 128
    q = np.full((M, K), 127, dtype=np.int8)
    q[1::2] = -127
    w = np.full((N, K), -128, dtype=np.int8)
    w[:, 128:256] = 127
    acc_g = cider.cider_test_gemm_i32_grouped(dev(q), dev(w), gs)
    np.testing.assert_array_equal(acc_g.cpu().numpy(), oracle.gemm_i32_grouped(q, w, gs))


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(300, 520, 2560), (257, 264, 1280), (520, 1032, 4096)])
def test_linear_pg_ragged(M, N, K, gs):
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=M + N + K + gs)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=M + K), gs)
    y = cider.cider_w8a8_linear_pg(dev_bits(x, oracle.F16), dev(qw), _gmajor(sw), gs)
    check_y(y, oracle.linear_pg(x, qw, sw, gs), oracle.F16)


@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(300, 520, 2560), (130, 264, 192)])
def test_w4a8_linear_ragged(M, N, K, gs):
    if K % gs:
        pytest.skip("gs must divide K")
    cider.cider_set_small_m_threshold(4)
    x = act(M, K, seed=M + N + K + 3 * gs)
    wp, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, seed=K + 7), gs)
    y = cider.cider_w4a8_linear_pg(dev_bits(x, oracle.F16), dev(wp), _gmajor(sw), gs)
    check_y(y, oracle.w4a8_linear_pg(x, wp, sw, gs), oracle.F16)


# ---------------------------------------------------------------- split K

@pytest.fixture
def split_k():
    yield cider.cider_test_set_split_k
    cider.cider_test_set_split_k(0)


@pytest.mark.parametrize("splits", [2, 3, 7])
@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(130, 264, 1280), (64, 136, 192), (257, 8, 2560)])
def test_gemm_i32_grouped_split_pieces(split_k, splits, gs, M, N, K):
    """Forced K pieces: every (tile, piece) unit writes its own groups'
    partials, so the result is the same bit for bit (K = 192 at gs = 64 leaves
    the last 128-wide block with one group; K = 192 has only 2 blocks, so 3
    and 7 pieces collapse to 2)."""
    if K % gs:
        pytest.skip("gs must divide K")
    split_k(splits)
    q, w = _codes(M, N, K, seed=7 * M + N + K + gs + splits)
    acc_g = cider.cider_test_gemm_i32_grouped(dev(q), dev(w), gs)
    np.testing.assert_array_equal(acc_g.cpu().numpy(), oracle.gemm_i32_grouped(q, w, gs))


@pytest.mark.parametrize("splits", [0, 2, 5])
@pytest.mark.parametrize("gs", [64, 128])
@pytest.mark.parametrize("M,N,K", [(128, 2560, 10240), (40, 264, 2560), (300, 520, 1280), (1024, 2560, 4096)])
def test_linear_pg_split(split_k, splits, gs, M, N, K):
    """Per-group linear with automatic (0) or forced K pieces: fp32 piece sums
    added by the reduce kernel, then scale_x and rounding.  At 1024 x 2560 the
    automatic plan runs 148 whole tiles and splits the 12 tiles of the tail
    round (rows 512.., columns 2304..), so both kinds of unit are checked."""
    cider.cider_set_small_m_threshold(4)
    split_k(splits)
    x = act(M, K, seed=M + N + K + gs + splits)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=N + K), gs)
    y = cider.cider_w8a8_linear_pg(dev_bits(x, oracle.F16), dev(qw), _gmajor(sw), gs)
    rows = np.arange(0, M, max(1, M // 40))
    check_y(y, oracle.linear_pg(x[rows], qw, sw, gs), oracle.F16, rows=rows)


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_w4a8_linear_split(split_k, dt):
    M, N, K, gs = 128, 1032, 4096, 64
    split_k(0)
    x = act(M, K, seed=77, dt=dt)
    wp, sw = oracle.quantize_weight_int4_pg(synth.weights(N, K, seed=78), gs)
    y = cider.cider_w4a8_linear_pg(dev_bits(x, dt), dev(wp), _gmajor(sw), gs)
    check_y(y, oracle.w4a8_linear_pg(x, wp, sw, gs, xdt=dt, ydt=dt), dt)


def test_split_needs_the_larger_workspace(split_k):
    """A workspace of cider_workspace_bytes(M, K) runs the unsplit kernel; one
    of cider_workspace_bytes_mnk(M, N, K) splits K; both give the oracle's
    answer, and the automatic split is > 1 for this shape (20 tiles)."""
    M, N, K, gs = 128, 2560, 10240, 128
    assert cider.cider_workspace_bytes_mnk(M, N, K) > cider.cider_workspace_bytes(M, K)
    x = act(M, K, seed=5)
    qw, sw = oracle.quantize_weight_pg(synth.weights(N, K, seed=6), gs)
    xd, wd, sd = dev_bits(x, oracle.F16), dev(qw), _gmajor(sw)
    small = torch.empty((cider.cider_workspace_bytes(M, K),), dtype=torch.uint8, device="cuda")
    big = torch.empty((cider.cider_workspace_bytes_mnk(M, N, K),), dtype=torch.uint8, device="cuda")
    y_plain = cider.cider_w8a8_linear_pg(xd, wd, sd, gs, workspace=small)
    y_split = cider.cider_w8a8_linear_pg(xd, wd, sd, gs, workspace=big)
    rows = np.arange(0, M, 5)
    ref = oracle.linear_pg(x[rows], qw, sw, gs)
    check_y(y_plain, ref, oracle.F16, rows=rows)
    check_y(y_split, ref, oracle.F16, rows=rows)
