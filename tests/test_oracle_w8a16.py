"""Pins of the oracle's W8A16 decode modes (Cider README, section "Metal Kernel
流水线", Decode: a direct INT8 matrix-vector product, weights dequantized on
the fly, no activation quantization): per channel y = round(scale_w[n] *
sum_k x[m,k] * w[n,k]); per group (the per-group INT8 MV kernel of the same
decode path) y = round(sum_g scale_w[n,g] * sum_{k in g} x[m,k] * w[n,k]).
Checked against hand-worked examples, exact rationals on tiny shapes, the
per-channel mode (one group spanning K) and the W8A8 modes where activation
quantization is exact."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.test_oracle_bruteforce import _nearest_f16


def test_w8a16_worked_example():
    # x = [1, 2, -0.5, 4] (fp16, exact)
    # row 0: w = [1, -2, 4, 3],     1 - 4 - 2 + 12 = 7,    7 * 0.5  = 3.5
    # row 1: w = [127, 0, -128, 1], 127 + 0 + 64 + 4 = 195, 195 * 0.25 = 48.75
    x = np.array([[1.0, 2.0, -0.5, 4.0]], dtype=np.float16)
    w = np.array([[1, -2, 4, 3], [127, 0, -128, 1]], dtype=np.int8)
    sw = np.array([0.5, 0.25], dtype=np.float32)
    y = oracle.as_float(oracle.w8a16_linear_pc(x.view(np.uint16), w, sw), oracle.F16)
    np.testing.assert_array_equal(y, [[3.5, 48.75]])


@pytest.mark.parametrize("seed", range(4))
def test_w8a16_bruteforce(seed):
    rng = np.random.default_rng(300 + seed)
    M, N, K = int(rng.integers(1, 4)), int(rng.integers(1, 6)), int(rng.integers(1, 12))
    x = rng.normal(0, 2, size=(M, K)).astype(np.float16)
    w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random(N) * 0.05 + 0.001).astype(np.float32)
    y = oracle.w8a16_linear_pc(x.view(np.uint16), w, sw).view(np.float16)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[m, k])) * int(w[n, k]) for k in range(K)) * Fraction(float(sw[n]))
            assert float(y[m, n]) == _nearest_f16(exact), (m, n)


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_w8a16_equals_w8a8_when_quantization_is_exact(dt):
    """x = codes * 2^j with one code of magnitude 127 per row: scale_x = 2^j
    and the codes come back unchanged, so the W8A8 linear (quantize, integer
    product, dequant) and the W8A16 product are the same number."""
    rng = np.random.default_rng(7)
    M, N, K = 3, 5, 64
    codes = rng.integers(-127, 128, size=(M, K))
    codes[:, 5] = 127 * np.array([1, -1, 1])
    x = codes * np.array([[2.0 ** -3], [2.0 ** 2], [1.0]])
    bits = oracle.narrow(x, dt)  # exact: |codes| <= 127 fits both formats
    np.testing.assert_array_equal(oracle.widen(bits, dt), x)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random(N) * 0.02 + 0.001).astype(np.float32)
    q, sx = oracle.quantize_act(bits, dt)
    np.testing.assert_array_equal(q, codes)
    np.testing.assert_array_equal(oracle.w8a16_linear_pc(bits, w, sw, xdt=dt, ydt=dt),
                                  oracle.linear_pc(bits, w, sw, xdt=dt, ydt=dt))


# ---- per-group scales (the per-group INT8 MV kernel of the pages' decode path)

def test_w8a16_pg_worked_example():
    # x = [1, 2, -0.5, 4] (fp16, exact), gs = 2 (two groups per row)
    # row 0: w = [1, -2 | 4, 3],      sw = [0.5, 0.25]
    #   group 0: 1*1 + 2*(-2) = -3, * 0.5 = -1.5;  group 1: -0.5*4 + 4*3 = 10, * 0.25 = 2.5
    #   y = -1.5 + 2.5 = 1.0
    # row 1: w = [127, 0 | -128, 1],  sw = [0.125, 2]
    #   group 0: 127 * 0.125 = 15.875;  group 1: 64 + 4 = 68, * 2 = 136
    #   y = 151.875 (exact in fp16: spacing 0.125 in [128, 256))
    x = np.array([[1.0, 2.0, -0.5, 4.0]], dtype=np.float16)
    w = np.array([[1, -2, 4, 3], [127, 0, -128, 1]], dtype=np.int8)
    sw = np.array([[0.5, 0.25], [0.125, 2.0]], dtype=np.float32)
    y = oracle.as_float(oracle.w8a16_linear_pg(x.view(np.uint16), w, sw, 2), oracle.F16)
    np.testing.assert_array_equal(y, [[1.0, 151.875]])


@pytest.mark.parametrize("seed", range(5))
def test_w8a16_pg_bruteforce(seed):
    rng = np.random.default_rng(400 + seed)
    gs = int(rng.integers(1, 4))
    M, N, G = int(rng.integers(1, 4)), int(rng.integers(1, 6)), int(rng.integers(1, 5))
    K = gs * G
    x = rng.normal(0, 2, size=(M, K)).astype(np.float16)
    w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random((N, G)) * 0.05 + 0.001).astype(np.float32)
    y = oracle.w8a16_linear_pg(x.view(np.uint16), w, sw, gs).view(np.float16)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(sw[n, g])) *
                        sum(Fraction(float(x[m, k])) * int(w[n, k]) for k in range(g * gs, (g + 1) * gs))
                        for g in range(G))
            assert float(y[m, n]) == _nearest_f16(exact), (m, n)


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_w8a16_pg_with_one_group_is_the_per_channel_product(dt):
    rng = np.random.default_rng(11)
    M, N, K = 3, 7, 96
    x = oracle.narrow(rng.normal(0, 1, size=(M, K)), dt)
    w = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random(N) * 0.02 + 0.001).astype(np.float32)
    np.testing.assert_array_equal(oracle.w8a16_linear_pg(x, w, sw[:, None], K, xdt=dt, ydt=dt),
                                  oracle.w8a16_linear_pc(x, w, sw, xdt=dt, ydt=dt))


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_w8a16_pg_equals_w8a8_pg_when_quantization_is_exact(dt):
    """x = codes * 2^j (one code of magnitude 127 per row): the W8A8 per-group
    linear sees the same products, and a power-of-two scale commutes exactly
    with every fp64 operation, so both modes give the same bits."""
    rng = np.random.default_rng(9)
    M, N, K, gs = 3, 5, 256, 64
    codes = rng.integers(-127, 128, size=(M, K))
    codes[:, 3] = 127 * np.array([1, -1, 1])
    x = codes * np.array([[2.0 ** -4], [2.0 ** 1], [1.0]])
    bits = oracle.narrow(x, dt)
    np.testing.assert_array_equal(oracle.widen(bits, dt), x)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sw = (rng.random((N, K // gs)) * 0.02 + 0.001).astype(np.float32)
    np.testing.assert_array_equal(oracle.w8a16_linear_pg(bits, w, sw, gs, xdt=dt, ydt=dt),
                                  oracle.linear_pg(bits, w, sw, gs, xdt=dt, ydt=dt))
