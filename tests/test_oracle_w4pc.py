"""Pins of the oracle's W4A8 linear with per-output-channel scales (Cider
README, table "量化": W4A8 weights symmetric INT4 with zero point 8, "per
column"): one scale max|W[n,:]|/7 per output channel, y = round(acc *
scale_x * scale_w[n]).  Checked against a hand-worked example, the W8A8
per-channel oracle on the unpacked weights, exact rationals, and the
quantizer's invariants."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.test_oracle_bruteforce import _nearest_f16


def test_w4pc_worked_example():
    # row 0: amax 7 -> scale 1: 3.5 -> 4 (half away), -7, 1.25 -> 1, 0
    # row 1: amax 14 -> scale 2: 7, -1.25 -> -1, 2.5 -> 3 (half away), 0.5 -> 1
    W = np.array([[3.5, -7.0, 1.25, 0.0], [14.0, -2.5, 5.0, 1.0]], np.float32)
    packed, sw = oracle.quantize_weight_int4_pc(W)
    np.testing.assert_array_equal(sw, [1.0, 2.0])
    # nibble = q + 8, even k in the low nibble: [12, 1 | 9, 8] and [15, 7 | 11, 9]
    np.testing.assert_array_equal(packed, [[0x1C, 0x89], [0x7F, 0x9B]])
    np.testing.assert_array_equal(oracle.unpack_int4(packed, 4), [[4, -7, 1, 0], [7, -1, 3, 1]])
    # x = [2, -1, 3, 127]: scale_x = 1, codes = x
    # acc0 = 8 + 7 + 3 + 0 = 18 -> 18;  acc1 = 14 + 1 + 9 + 127 = 151 -> 151 * 2 = 302
    x = np.array([[2.0, -1.0, 3.0, 127.0]], np.float16)
    y = oracle.as_float(oracle.w4a8_linear_pc(x.view(np.uint16), packed, sw), oracle.F16)
    np.testing.assert_array_equal(y, [[18.0, 302.0]])


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_w4pc_equals_w8a8_pc_on_unpacked_weights(dt):
    rng = np.random.default_rng(21)
    M, N, K = 5, 24, 256
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    packed, sw = oracle.quantize_weight_int4_pc(W)
    x = oracle.narrow(rng.normal(0, 1, size=(M, K)), dt)
    np.testing.assert_array_equal(oracle.w4a8_linear_pc(x, packed, sw, xdt=dt, ydt=dt),
                                  oracle.linear_pc(x, oracle.unpack_int4(packed, K), sw, xdt=dt, ydt=dt))


def test_w4pc_quantizer_invariants():
    rng = np.random.default_rng(3)
    W = rng.standard_t(3, size=(16, 512)).astype(np.float32)
    W[5] = 0.0
    packed, sw = oracle.quantize_weight_int4_pc(W)
    q = oracle.unpack_int4(packed, 512)
    assert q.min() >= -8 and q.max() <= 7
    amax = np.abs(W).max(axis=1)
    np.testing.assert_array_equal(sw, amax / np.float32(7))
    assert not q[5].any() and sw[5] == 0
    for n in range(16):
        if n != 5:
            k = int(np.argmax(np.abs(W[n])))
            assert q[n, k] == 7 * np.sign(W[n, k])


@pytest.mark.parametrize("seed", range(4))
def test_w4pc_bruteforce_rationals(seed):
    rng = np.random.default_rng(700 + seed)
    M, N, K = int(rng.integers(1, 3)), int(rng.integers(1, 4)), 2 * int(rng.integers(1, 6))
    W = rng.normal(0, 1, size=(N, K)).astype(np.float32)
    x = rng.normal(0, 2, size=(M, K)).astype(np.float16)
    packed, sw = oracle.quantize_weight_int4_pc(W)
    w = oracle.unpack_int4(packed, K)
    q, sx = oracle.quantize_act(x.view(np.uint16), oracle.F16)
    y = oracle.w4a8_linear_pc(x.view(np.uint16), packed, sw).view(np.float16)
    for m in range(M):
        for n in range(N):
            acc = sum(int(q[m, k]) * int(w[n, k]) for k in range(K))
            exact = acc * Fraction(float(sx[m])) * Fraction(float(sw[n]))
            assert float(y[m, n]) == _nearest_f16(exact), (m, n)
