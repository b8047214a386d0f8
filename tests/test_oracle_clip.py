"""Pins of the oracle's percentile-clipped weight scales (Cider README,
section "说明": scales by min-max by default, or by a percentile method,
clip_percentile=99.9).

Reading: the clipping value c of a slab (an output row, or one group of gs
along K) is the p-th percentile of its magnitudes |w| -- linear
interpolation at position p/100 * (len-1) of the ascending order -- with
scale = c / 127 and codes clipped symmetrically to [-127, 127]; a slab whose
percentile is 0 falls back to max|w|.

Checked against hand-worked rows, numpy's percentile (an independent fp64
implementation of the same definition), exact rationals on tiny rows, the
p = 100 case (the maximum, i.e. min-max), and the quantization error bound.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _f32(x):
    return np.float32(x)


def test_clip_pc_worked_example_p90():
    # |w| ascending: 0 1 2 3 4 5 6 7 8 9 20; p = 90 -> position 0.9 * 10 = 9 -> c = 9
    w = np.array([[0, 1, -2, 3, 4, -5, 6, 7, 8, 9, -20]], np.float32)
    q, s = oracle.quantize_weight_pc_clip(w, 90.0)
    assert s[0] == _f32(9) / _f32(127)
    # w * 127 / 9: 0, 14.1, -28.2, 42.3, 56.4, -70.6, 84.7, 98.8, 112.9, 127, -282.2 (clipped)
    np.testing.assert_array_equal(q[0], [0, 14, -28, 42, 56, -71, 85, 99, 113, 127, -127])


def test_clip_pc_worked_example_interpolated():
    # p = 95 -> position 9.5: c = 9 + 0.5 * (20 - 9) = 14.5
    w = np.array([[0, 1, -2, 3, 4, -5, 6, 7, 8, 9, -20]], np.float32)
    q, s = oracle.quantize_weight_pc_clip(w, 95.0)
    assert s[0] == _f32(14.5) / _f32(127)
    # w * 127 / 14.5: 1 -> 8.76, -2 -> -17.5 (17.517), 4 -> 35.03, -5 -> -43.79, 9 -> 78.83, -20 -> -175.2
    np.testing.assert_array_equal(q[0], [0, 9, -18, 26, 35, -44, 53, 61, 70, 79, -127])


def test_clip_pg_worked_example():
    # two groups of 4, p = 50 -> position 1.5: c0 = 2 + 0.5 * 1 = 2.5, c1 = 20 + 0.5 * 10 = 25
    w = np.array([[1, 2, 3, 4, 10, -20, 30, 40]], np.float32)
    q, s = oracle.quantize_weight_pg_clip(w, 4, 50.0)
    np.testing.assert_array_equal(s[0], [_f32(2.5) / _f32(127), _f32(25) / _f32(127)])
    # group 0: 50.8, 101.6, 152.4 -> 127, 203 -> 127; group 1: 50.8, -101.6, 152.4, 203
    np.testing.assert_array_equal(q[0], [51, 102, 127, 127, 51, -102, 127, 127])


def test_clip_zero_percentile_falls_back_to_max():
    w = np.zeros((1, 1000), np.float32)
    w[0, 123] = 5.0
    q, s = oracle.quantize_weight_pc_clip(w, 99.0)  # position 989.01: both neighbours are 0
    assert s[0] == _f32(5) / _f32(127)
    assert q[0, 123] == 127 and np.count_nonzero(q) == 1
    qz, sz = oracle.quantize_weight_pc_clip(np.zeros((2, 64), np.float32), 99.9)
    assert not qz.any() and not sz.any()


def test_percentile_position():
    assert oracle.percentile_position(100.0, 64) == (63, 0.0)
    assert oracle.percentile_position(0.0, 64) == (0, 0.0)
    assert oracle.percentile_position(50.0, 5) == (2, 0.0)
    i, t = oracle.percentile_position(99.9, 2560)  # 0.999 * 2559 = 2556.441
    assert i == 2556 and abs(float(t) - 0.441) < 1e-6
    assert oracle.percentile_position(99.9, 1) == (0, 0.0)


@pytest.mark.parametrize("p", [99.9, 99.0, 90.0, 50.0])
def test_clip_scales_match_numpy_percentile(p):
    rng = np.random.default_rng(int(p * 10))
    W = rng.standard_t(3, size=(8, 2560)).astype(np.float32)  # heavy tails: outliers to clip
    _, s = oracle.quantize_weight_pc_clip(W, p)
    ref = np.percentile(np.abs(W).astype(np.float64), p, axis=1) / 127.0
    np.testing.assert_allclose(s, ref, rtol=1e-6)
    gs = 64
    _, sg = oracle.quantize_weight_pg_clip(W, gs, p)
    refg = np.percentile(np.abs(W).astype(np.float64).reshape(8, -1, gs), p, axis=2) / 127.0
    np.testing.assert_allclose(sg, refg, rtol=1e-6)


@pytest.mark.parametrize("seed", range(6))
def test_clip_bruteforce_rationals(seed):
    rng = np.random.default_rng(500 + seed)
    for p in (0.0, 12.5, 50.0, 90.0, 99.9, 100.0):
        n = int(rng.integers(1, 10))
        w = rng.integers(-40, 41, size=(1, n)).astype(np.float32)
        _, s = oracle.quantize_weight_pc_clip(w, p)
        a = sorted(abs(int(v)) for v in w[0])
        pos = Fraction(str(p)) / 100 * (n - 1)
        i = int(pos)
        v = Fraction(a[i]) + (pos - i) * (a[i + 1] - a[i]) if i + 1 < n else Fraction(a[i])
        c = v if v != 0 else Fraction(max(a))
        exact = c / 127
        assert abs(Fraction(float(s[0])) - exact) <= 4 * Fraction(float(np.spacing(np.float32(exact)))), (p, a)


@pytest.mark.parametrize("gs", [0, 64, 128])
def test_clip_at_100_equals_min_max(gs):
    W = np.random.default_rng(gs).normal(size=(16, 1024)).astype(np.float32)
    if gs == 0:
        q, s = oracle.quantize_weight_pc_clip(W, 100.0)
        q0, s0 = oracle.quantize_weight_pc(W)
    else:
        q, s = oracle.quantize_weight_pg_clip(W, gs, 100.0)
        q0, s0 = oracle.quantize_weight_pg(W, gs)
    np.testing.assert_array_equal(s, s0)
    np.testing.assert_array_equal(q, q0)


def test_clip_error_bound_and_saturation():
    rng = np.random.default_rng(11)
    W = rng.standard_t(2, size=(6, 4096)).astype(np.float32)
    q, s = oracle.quantize_weight_pc_clip(W, 99.9)
    assert q.min() >= -127 and q.max() <= 127
    c = s.astype(np.float64) * 127
    inside = np.abs(W) <= c[:, None] * (1 - 1e-6)
    err = np.abs(q.astype(np.float64) * s[:, None] - W)
    assert np.all(err[inside] <= (s[:, None] * (0.5 + 1e-5)).repeat(W.shape[1], 1)[inside])
    outside = np.abs(W) > c[:, None] * (1 + 1e-6)
    assert outside.any()
    np.testing.assert_array_equal(q[outside], 127 * np.sign(W[outside]).astype(np.int8))
