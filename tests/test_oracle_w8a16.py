"""Pins of the oracle's W8A16 decode mode (Cider README, section "Metal Kernel
流水线", Decode: a direct INT8 matrix-vector product, weights dequantized on
the fly, no activation quantization): y = round(scale_w[n] * sum_k x[m,k] *
w[n,k]).  Checked against a hand-worked example, exact rationals on tiny
shapes, and the W8A8 mode where activation quantization is exact."""
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
