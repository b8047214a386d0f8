"""Pins of the decode-attention oracle (Cider README, section "优化 SDPA
（解码注意力）": Q_seq = 1, no mask, grouped KV heads, D = 128): against
PyTorch's own scaled_dot_product_attention in float64 (an independent
implementation), and closed forms that a wrong scale, a wrong KV-head index,
a missing max shift or a transposed product would break."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import sdpa

D = 128


def _bits(a, dt=oracle.F16):
    return oracle.narrow(np.asarray(a, np.float64), dt)


def _rand(shape, seed, scale=1.0, dt=oracle.F16):
    return _bits(np.random.default_rng(seed).normal(0, scale, size=shape), dt)


@pytest.mark.parametrize("H_q,H_kv,N", [(32, 32, 64), (32, 8, 300), (32, 4, 1025), (8, 1, 7)])
@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_sdpa_matches_torch_f64(H_q, H_kv, N, dt):
    q, k, v = _rand((H_q, D), 1, dt=dt), _rand((H_kv, N, D), 2, dt=dt), _rand((H_kv, N, D), 3, dt=dt)
    ours = sdpa.sdpa_decode_f64(q, k, v, dt)
    G = H_q // H_kv
    qt = torch.from_numpy(oracle.widen(q, dt).astype(np.float64))[None, :, None, :]
    kt = torch.from_numpy(oracle.widen(k, dt).astype(np.float64)).repeat_interleave(G, 0)[None]
    vt = torch.from_numpy(oracle.widen(v, dt).astype(np.float64)).repeat_interleave(G, 0)[None]
    ref = F.scaled_dot_product_attention(qt, kt, vt)[0, :, 0, :].numpy()
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_sdpa_single_key_returns_its_value_exactly():
    q, k, v = _rand((8, D), 4), _rand((2, 1, D), 5), _rand((2, 1, D), 6)
    out = sdpa.sdpa_decode(q, k, v)
    np.testing.assert_array_equal(out[:4], np.repeat(v[0], 4, axis=0))
    np.testing.assert_array_equal(out[4:], np.repeat(v[1], 4, axis=0))


def test_sdpa_zero_query_is_the_mean_of_values():
    q = _bits(np.zeros((4, D)))
    k, v = _rand((4, 50, D), 7, scale=3.0), _rand((4, 50, D), 8)
    out = sdpa.sdpa_decode_f64(q, k, v)
    np.testing.assert_allclose(out, oracle.widen(v, oracle.F16).astype(np.float64).mean(axis=1), rtol=0, atol=1e-15)


def test_sdpa_two_keys_closed_form_fixes_the_scale():
    # s0 = x * a / sqrt(D), s1 = 0: out = sigmoid(s0) * v0 + (1 - sigmoid(s0)) * v1
    x, a = 2.0, 3.0
    q = np.zeros((1, D)); q[0, 0] = x
    k = np.zeros((1, 2, D)); k[0, 0, 0] = a
    v = np.zeros((1, 2, D)); v[0, 0, :] = 1.0; v[0, 1, :] = -0.5
    out = sdpa.sdpa_decode_f64(_bits(q), _bits(k), _bits(v))
    p0 = 1.0 / (1.0 + math.exp(-x * a / math.sqrt(D)))
    np.testing.assert_allclose(out[0], p0 * 1.0 + (1 - p0) * -0.5, rtol=1e-14)


def test_sdpa_kv_head_of_each_query_head():
    # H_q = 6, H_kv = 3: query heads 2h and 2h+1 read KV head h.  Give KV head h
    # constant values h + 1: every output of a query head is then its KV head's constant.
    H_q, H_kv, N = 6, 3, 40
    q, k = _rand((H_q, D), 9), _rand((H_kv, N, D), 10)
    v = _bits(np.stack([np.full((N, D), h + 1.0) for h in range(H_kv)]))
    out = sdpa.sdpa_decode_f64(q, k, v)
    np.testing.assert_allclose(out, np.repeat(np.arange(1.0, H_kv + 1)[:, None], 2, axis=0) * np.ones((1, D)),
                               rtol=0, atol=1e-13)  # the weights sum to 1 up to fp64 rounding


def test_sdpa_large_scores_need_the_max_shift():
    # scores near 700 overflow exp() without the shift; the dominant key wins
    q = np.zeros((1, D)); q[0, :] = 2.0
    k = np.zeros((1, 3, D)); k[0, 0, :] = 100.0; k[0, 1, :] = 99.0; k[0, 2, :] = -5.0
    v = np.zeros((1, 3, D)); v[0, 0, :] = 1.0; v[0, 1, :] = 2.0; v[0, 2, :] = 3.0
    out = sdpa.sdpa_decode_f64(_bits(q), _bits(k), _bits(v))
    s = np.array([200.0 * D, 198.0 * D, -10.0 * D]) / math.sqrt(D)
    p = np.exp(s - s.max()); p /= p.sum()
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0], p @ np.array([1.0, 2.0, 3.0]), rtol=1e-14)


MUTATIONS = {
    "scale_dropped": ("/ np.sqrt(D)", ""),
    "kv_head_by_modulo": ("g = h // G", "g = h % H_kv"),
    "max_shift_dropped": ("np.exp(s - s.max())", "np.exp(s)"),
    "values_reversed": ("(e / e.sum()) @ vf[g]", "(e / e.sum()) @ vf[g][::-1]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    """A copy of the oracle with one plausible mistake must fail a pin."""
    old, new = MUTATIONS[name]
    src = open(sdpa.__file__).read()
    assert src.count(old) == 1
    ns = {"np": np, "F16": oracle.F16, "narrow": oracle.narrow, "widen": oracle.widen}
    exec(compile(src.replace(old, new).replace("from . import F16, narrow, widen", ""), "mutant", "exec"), ns)
    monkeypatch.setattr(sdpa, "sdpa_decode_f64", ns["sdpa_decode_f64"])
    monkeypatch.setattr(sdpa, "sdpa_decode", ns["sdpa_decode"])
    pins = [test_sdpa_two_keys_closed_form_fixes_the_scale, test_sdpa_kv_head_of_each_query_head,
            test_sdpa_large_scores_need_the_max_shift, lambda: test_sdpa_matches_torch_f64(32, 8, 300, oracle.F16)]
    failures = 0
    for pin in pins:
        try:
            with np.errstate(all="ignore"):
                pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught {name}"
