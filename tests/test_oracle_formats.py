"""Pin the oracle's number-format helpers to library routines and to exact arithmetic.

* fp16 -> fp32 widening: all 65536 bit patterns against numpy's float16.
* bf16 -> fp32 widening: all 65536 bit patterns against torch's bfloat16.
* fp64 -> fp16 rounding: against numpy's float64 -> float16 cast (round to
  nearest even), on random values, ties, subnormals and overflow.
* fp32 -> bf16 rounding: against torch's float32 -> bfloat16 cast.
* round-half-away-from-zero: against Python's decimal ROUND_HALF_UP (which
  rounds halfway cases away from zero) on exact float32 values.
"""
from decimal import ROUND_HALF_UP, Decimal

import numpy as np
import torch

import oracle


def test_f16_widen_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits, oracle.F16)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_widen_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits, oracle.BF16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _f16_specials():
    f16 = np.arange(0, 0x7C01, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = (f16[:-1] + f16[1:]) / 2.0          # exact ties between neighbours
    near = np.nextafter(mids, np.inf)
    below = np.nextafter(mids, -np.inf)
    big = np.array([65504.0, 65519.99, 65520.0, 65536.0, 1e6, np.inf])
    v = np.concatenate([f16, mids, near, below, big])
    return np.concatenate([v, -v])


def test_f64_to_f16_against_numpy():
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.standard_normal(200_000) * s for s in (1e-6, 1e-3, 1.0, 1e3, 6e4)])
    v = np.concatenate([_f16_specials(), rand, [0.0, -0.0]])
    ours = oracle.narrow(v, oracle.F16)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_f32_to_bf16_against_torch():
    rng = np.random.default_rng(1)
    v32 = np.concatenate([
        rng.standard_normal(300_000).astype(np.float32) * np.float32(s) for s in (1e-30, 1e-3, 1.0, 1e30)
    ])
    # exact ties: bf16 neighbours' midpoints are float32 values
    b = rng.integers(0, 0x7F7F, 100_000, dtype=np.uint32)
    ties = ((b << 16) | 0x8000).view(np.float32)
    v32 = np.concatenate([v32, ties, -ties, np.float32([3.4e38, 3.39e38, 1e-45])])
    ours = oracle.narrow(v32.astype(np.float64), oracle.BF16)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_round_half_away_against_decimal():
    rng = np.random.default_rng(2)
    halves = (np.arange(-300, 301) / 2.0).astype(np.float32)
    tricky = np.float32([0.49999997, -0.49999997, 0.5, -0.5, 1.5, 2.5, -2.5, 126.5, -127.5,
                         8388607.5, 8388608.0, 1e10, 0.0, -0.0, 1.4e-45])
    rand = (rng.standard_normal(50_000) * 100).astype(np.float32)
    t = np.concatenate([halves, tricky, rand])
    ours = oracle.round_half_away(t)
    ref = np.array([float(Decimal(float(v)).quantize(Decimal(1), rounding=ROUND_HALF_UP)) for v in t],
                   dtype=np.float32)
    np.testing.assert_array_equal(ours, ref)
    assert oracle.round_half_away([0.49999997])[0] == 0.0  # floor(|t| + 0.5) would give 1
