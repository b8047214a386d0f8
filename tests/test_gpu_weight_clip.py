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
