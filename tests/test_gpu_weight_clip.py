"""The percentile-clipped weight quantizers (Cider README, section "说明",
clip_percentile) against the oracle, bit for bit: every scale (as fp32 bits)
and every code, per channel and per group of 64 / 128, at the full weight
shapes of the benchmarked linears and on ragged, tied, zero and tiny
slabs."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_activation_quantized_b200 as cider
from tests.parity import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_device_status()


def _heavy(N, K, seed):
    """Student-t(3) weights: heavy tails, so a percentile below 100 clips."""
    return np.random.default_rng(seed).standard_t(3, size=(N, K)).astype(np.float32) * 0.02


def _check_pc(W, p):
    w, s = cider.cider_quantize_weight_pc_clip(dev(W), p)
    qo, so = oracle.quantize_weight_pc_clip(W, p)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(w.cpu().numpy(), qo)


def _check_pg(W, gs, p):
    w, s = cider.cider_quantize_weight_pg_clip(dev(W), gs, p)
    qo, so = oracle.quantize_weight_pg_clip(W, gs, p)
    np.testing.assert_array_equal(s.cpu().numpy().T.view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(w.cpu().numpy(), qo)


@pytest.mark.parametrize("N,K", [(10240, 2560), (2560, 10240)])
def test_clip_pc_full_shapes(N, K):
    _check_pc(_heavy(N, K, seed=N + K), 99.9)


@pytest.mark.parametrize("gs", [64, 128])
def test_clip_pg_full_shape(gs):
    _check_pg(_heavy(2560, 10240, seed=gs), gs, 99.9)


@pytest.mark.parametrize("p", [0.0, 50.0, 99.0, 99.9, 100.0])
@pytest.mark.parametrize("N,K", [(1, 1), (3, 17), (7, 1000), (33, 4097)])
def test_clip_pc_ragged(N, K, p):
    _check_pc(_heavy(N, K, seed=N * K + int(p)), p)


@pytest.mark.parametrize("p", [0.0, 37.5, 99.9, 100.0])
@pytest.mark.parametrize("gs", [64, 128])
def test_clip_pg_ragged(gs, p):
    _check_pg(_heavy(5, 3 * gs, seed=gs + int(p)), gs, p)


def _p_for_rank_from_top(length, j):
    """A percentile whose first order statistic is rank j counted from the top
    (k0 = length - 1 - j) with interpolation weight 1/2 (100 for j = 0)."""
    return 100.0 if j == 0 else 100.0 * (length - 1 - j + 0.5) / (length - 1)


@pytest.mark.parametrize("j", [0, 1, 2, 12, 13, 40])
@pytest.mark.parametrize("K", [1001, 5000])
def test_clip_pc_ranks_from_top(K, j):
    """Ranks j <= 12 from the top take the walk down the distinct magnitudes,
    larger ranks the counting passes; rows of up to 4096 weights sit in
    registers, longer ones are read through L1.  Each must give the oracle's
    scales and codes, with long runs of equal magnitudes and a tied floor."""
    rng = np.random.default_rng(K + j)
    W = _heavy(6, K, seed=K * 7 + j)
    W[1] = rng.integers(-4, 5, size=K).astype(np.float32)
    W[2, :] = 0.5
    W[2, :3] = [3.0, -3.0, 2.0]
    W[3, :] = -0.0
    W[3, 5] = 1.0
    _check_pc(W, _p_for_rank_from_top(K, j))


@pytest.mark.parametrize("j", [0, 1, 12, 13, 30])
@pytest.mark.parametrize("gs", [64, 128])
def test_clip_pg_ranks_from_top(gs, j):
    rng = np.random.default_rng(gs + j)
    W = _heavy(5, 4 * gs, seed=gs * 3 + j)
    W[1] = rng.integers(-3, 4, size=4 * gs).astype(np.float32)
    W[2, :] = 0.25
    W[2, ::gs] = -1.0
    _check_pg(W, gs, _p_for_rank_from_top(gs, j))


def test_clip_ties_zeros_and_negative_zero():
    rng = np.random.default_rng(4)
    W = rng.integers(-3, 4, size=(6, 512)).astype(np.float32)  # many equal magnitudes
    W[1] = 0.0
    W[2] = -0.0
    W[3, :] = 0.0
    W[3, 17] = -2.5  # the 99th percentile is 0: min-max fallback
    W[4, ::2] = -0.0
    for p in (99.0, 99.9, 75.0):
        _check_pc(W, p)
        _check_pg(W, 64, p)
        _check_pg(W, 128, p)


def test_clip_100_equals_min_max_on_gpu():
    W = _heavy(96, 2048, seed=1)
    w, s = cider.cider_quantize_weight_pc_clip(dev(W), 100.0)
    w0, s0 = cider.cider_quantize_weight_pc(dev(W))
    assert torch.equal(w, w0) and torch.equal(s, s0)
    for gs in (64, 128):
        w, s = cider.cider_quantize_weight_pg_clip(dev(W), gs, 100.0)
        w0, s0 = cider.cider_quantize_weight_pg(dev(W), gs)
        assert torch.equal(w, w0) and torch.equal(s, s0)


def test_clip_argument_checks():
    W = dev(_heavy(4, 256, seed=2))
    for bad in (-0.5, 100.5, float("nan")):
        with pytest.raises(cider.CiderError):
            cider.cider_quantize_weight_pc_clip(W, bad)
    with pytest.raises(cider.CiderError):
        cider.cider_quantize_weight_pg_clip(W, 32, 99.9)
    with pytest.raises(cider.CiderError):
        cider.cider_quantize_weight_pg_clip(dev(_heavy(4, 200, seed=3)), 64, 99.9)


@pytest.mark.parametrize("K", [4, 12, 1020, 2048, 2052, 2556, 2560, 2564, 4092, 4096, 4100])
def test_clip_pc_row_per_warp_widths(K):
    """Rows with K % 4 == 0 and K <= 4096 on 16-byte aligned memory take one
    warp per row (K <= 2048, 2560 and 4096 are the three register widths);
    the same rows 4 bytes past a 16-byte boundary, and K = 4100, take the
    CTA-per-row kernels.  All bit for bit."""
    W = np.ascontiguousarray(_heavy(37, K, seed=K))
    for p in (99.9, 50.0):
        _check_pc(W, p)
        flat = torch.zeros(W.size + 1, dtype=torch.float32, device="cuda")
        flat[1:] = torch.from_numpy(W.ravel()).cuda()
        w, s = cider.cider_quantize_weight_pc_clip(flat[1:].view(W.shape), p)
        qo, so = oracle.quantize_weight_pc_clip(W, p)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
        np.testing.assert_array_equal(w.cpu().numpy(), qo)


def test_clip_pc_saturation_and_halfway_codes():
    """Codes computed through the reciprocal: values far beyond the clipped
    scale saturate at +-127, exact halfway quotients keep the oracle's
    rounding (half away from zero), and a zero row gives zero codes."""
    K = 1024
    W = np.zeros((4, K), dtype=np.float32)
    W[0] = np.linspace(-1.0, 1.0, K, dtype=np.float32)
    W[0, :8] = [1e3, -1e3, 5e2, -5e2, 3e38, -3e38, 1e-30, -1e-30]
    base = np.float32(127.0 / 64.0)
    W[1] = base
    W[1, :64] = (np.arange(64, dtype=np.float32) + np.float32(0.5)) * np.float32(1.0 / 64.0) * base
    W[1, 64] = np.float32(2.0) * base
    W[2] = 0.0
    W[3] = np.random.default_rng(9).standard_normal(K).astype(np.float32)
    for p in (99.9, 90.0, 50.0):
        _check_pc(W, p)
        _check_pg(W, 64, p)
