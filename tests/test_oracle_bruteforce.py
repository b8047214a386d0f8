"""Pin the oracle by brute force on tiny inputs, with exact rational arithmetic.

The brute force here does not follow the oracle's steps: the INT8 code is
found by searching all 256 candidates for the one nearest to the fp32
quotient (ties to the larger magnitude), the products are summed as Python
integers, and the fp16 output is the representable value nearest to the
exact rational result (ties to the even significand), found by comparing
neighbours as Fractions.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w8a8_activation_quantized_b200 import synth


def _nearest_code(t: float, lo: int, hi: int) -> int:
    tf = Fraction(t)
    best = None
    for c in range(lo, hi + 1):
        d = abs(tf - c)
        if best is None or d < best[0] or (d == best[0] and abs(c) > abs(best[1])):
            best = (d, c)
    return best[1]


def _nearest_f16(v: Fraction) -> float:
    """fp16 value nearest to the rational v, ties to even significand."""
    approx = np.float16(float(v))
    cands = {approx, np.nextafter(approx, np.float16(np.inf)), np.nextafter(approx, np.float16(-np.inf))}
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - v)
        even = (int(np.float16(c).view(np.uint16)) & 1) == 0
        if best is None or d < best[0] or (d == best[0] and even):
            best = (d, float(c))
    return best[1]


@pytest.mark.parametrize("seed", range(6))
def test_activation_codes_bruteforce(seed):
    rng = np.random.default_rng(seed)
    M, K = 3, 8
    x = (rng.standard_normal((M, K)) * rng.choice([0.01, 1, 300], size=(M, 1))).astype(np.float16)
    if seed == 0:
        x[1] = np.float16([2.5, -0.5, 0.5, 1.5, -127, 3.5, 0, 64])  # exact halves against max 127
    q, sx = oracle.quantize_act(x)
    for m in range(M):
        xs = x[m].astype(np.float32)
        amax = np.max(np.abs(xs))
        # the stored scale is the fp32 number nearest to amax/127
        assert abs(Fraction(float(sx[m])) - Fraction(float(amax)) / 127) <= \
            Fraction(float(np.spacing(np.float32(sx[m])))) / 2
        for k in range(K):
            t = np.float32(xs[k]) / sx[m]  # the fp32 quotient the codes are decided on
            assert q[m, k] == _nearest_code(float(t), -128, 127), (m, k, float(t))


@pytest.mark.parametrize("seed", range(4))
def test_linear_pc_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    M, N, K = int(rng.integers(1, 5)), int(rng.integers(1, 6)), int(rng.integers(1, 9))
    x = synth.activations(M, K, seed, outlier_frac=0.25)
    W = synth.weights(N, K, seed, std=0.5)
    qw, sw = oracle.quantize_weight_pc(W)
    # weight codes by search, too
    for n in range(N):
        for k in range(K):
            assert qw[n, k] == _nearest_code(float(np.float32(W[n, k]) / sw[n]), -128, 127)
    q, sx = oracle.quantize_act(x)
    y = oracle.linear_pc(x, qw, sw).view(np.float16)
    for m in range(M):
        for n in range(N):
            acc = sum(int(q[m, k]) * int(qw[n, k]) for k in range(K))
            exact = acc * Fraction(float(sx[m])) * Fraction(float(sw[n]))
            assert float(y[m, n]) == _nearest_f16(exact), (m, n)


@pytest.mark.parametrize("gs", [2, 4])
def test_linear_pg_bruteforce(gs):
    rng = np.random.default_rng(7 + gs)
    M, N, K = 3, 4, 8
    x = synth.activations(M, K, gs, outlier_frac=0.25)
    W = (rng.standard_normal((N, K)) * rng.choice([0.01, 1.0, 20.0], size=(N, K))).astype(np.float32)
    qw, sw = oracle.quantize_weight_pg(W, gs)
    q, sx = oracle.quantize_act(x)
    y = oracle.linear_pg(x, qw, sw, gs).view(np.float16)
    for m in range(M):
        for n in range(N):
            total = Fraction(0)
            for g in range(K // gs):
                acc = sum(int(q[m, k]) * int(qw[n, k]) for k in range(g * gs, (g + 1) * gs))
                total += acc * Fraction(float(sw[n, g]))
            exact = Fraction(float(sx[m])) * total
            assert float(y[m, n]) == _nearest_f16(exact), (m, n)


def test_int4_codes_bruteforce():
    rng = np.random.default_rng(5)
    N, K, gs = 3, 8, 4
    W = (rng.standard_normal((N, K)) * 0.1).astype(np.float32)
    W[0, :4] = np.float32([0.7, -0.25, 0.05, 0.35])  # 0.35/0.1 = 3.5 -> a tie (up to fp32 rounding)
    packed, sw = oracle.quantize_weight_int4_pg(W, gs)
    w = oracle.unpack_int4(packed, K)
    for n in range(N):
        for k in range(K):
            t = np.float32(W[n, k]) / sw[n, k // gs]
            assert w[n, k] == _nearest_code(float(t), -8, 7)
