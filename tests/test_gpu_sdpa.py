"""Decode attention on the GPU (Cider README, section "优化 SDPA（解码注意
力）") against the float64 oracle: the pages' configurations (MHA, GQA4, GQA8
at D = 128) up to N = 32K, ragged sequence lengths (one key, fewer keys than
a chunk's streams, chunk tails), other group sizes, bf16, and the argument
checks.

Tolerance: every output is a convex combination of its KV head's value rows,
so |out| <= max|V|; its final rounding costs at most one unit of the format
at that size and the fp32 chunked softmax adds far less.  The bound is four
units at max|V|: 2^-9 * max|V| for fp16, 2^-6 * max|V| for bf16."""
import numpy as np
import pytest
import torch

import oracle
from oracle import sdpa
import w8a8_activation_quantized_b200 as cider
from tests.parity import dev_bits, host_bits

pytestmark = pytest.mark.gpu
D = 128
TOL = {oracle.F16: 2.0 ** -9, oracle.BF16: 2.0 ** -6}


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    cider.cider_device_status()


def _inputs(H_q, H_kv, N, seed, dt=oracle.F16):
    rng = np.random.default_rng(seed)
    q = oracle.narrow(rng.normal(0, 1, size=(H_q, D)), dt)
    k = oracle.narrow(rng.normal(0, 1, size=(H_kv, N, D)), dt)
    v = oracle.narrow(rng.normal(0, 1, size=(H_kv, N, D)), dt)
    return q, k, v


def _check(H_q, H_kv, N, seed, dt=oracle.F16):
    q, k, v = _inputs(H_q, H_kv, N, seed, dt)
    out = cider.cider_sdpa_decode(dev_bits(q, dt), dev_bits(k, dt), dev_bits(v, dt))
    got = oracle.as_float(host_bits(out), dt).astype(np.float64)
    ref = oracle.as_float(sdpa.sdpa_decode(q, k, v, dt), dt).astype(np.float64)
    vmax = np.abs(oracle.widen(v, dt)).max(axis=(1, 2)).repeat(H_q // H_kv)[:, None]
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= TOL[dt] * vmax), f"max err / max|V| = {np.max(err / vmax):.3g}"
    return out


@pytest.mark.parametrize("H_kv", [32, 8, 4])
@pytest.mark.parametrize("N", [1024, 4096, 32768])
def test_sdpa_pages_configs(H_kv, N):
    _check(32, H_kv, N, seed=H_kv + N)


@pytest.mark.parametrize("N", [1, 2, 15, 16, 17, 77, 1025, 3001])
@pytest.mark.parametrize("H_q,H_kv", [(32, 8), (32, 32), (8, 1), (6, 3), (3, 1)])
def test_sdpa_ragged(H_q, H_kv, N):
    _check(H_q, H_kv, N, seed=N * 7 + H_q + H_kv)


@pytest.mark.parametrize("H_kv", [32, 4])
def test_sdpa_bf16(H_kv):
    _check(32, H_kv, 2049, seed=H_kv, dt=oracle.BF16)


def test_sdpa_single_key_is_its_value_exactly():
    q, k, v = _inputs(32, 8, 1, seed=5)
    out = cider.cider_sdpa_decode(dev_bits(q, oracle.F16), dev_bits(k, oracle.F16), dev_bits(v, oracle.F16))
    np.testing.assert_array_equal(host_bits(out), np.repeat(v[:, 0, :], 4, axis=0))


def test_sdpa_argument_checks():
    q, k, v = _inputs(32, 8, 64, seed=6)
    qd, kd, vd = (dev_bits(a, oracle.F16) for a in (q, k, v))
    with pytest.raises(cider.CiderError):  # H_kv must divide H_q
        cider.cider_sdpa_decode(dev_bits(_inputs(30, 8, 64, 1)[0], oracle.F16), kd, vd)
    with pytest.raises(cider.CiderError):  # D = 128 only
        cider.cider_sdpa_decode(qd[:, :64].contiguous(), kd[:, :, :64].contiguous(), vd[:, :, :64].contiguous())
    with pytest.raises(cider.CiderError):  # workspace too small
        cider.cider_sdpa_decode(qd, kd, vd, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
