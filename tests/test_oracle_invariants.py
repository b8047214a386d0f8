"""Pin the oracle with invariants and with special cases that reduce to library routines.

* |q| <= 127, and the largest-magnitude element of each token maps to +-127;
* q is unchanged when a token is scaled by 2^j (exact in fp16);
* an all-zero token gives scale 0, q = 0 and an all-zero output row;
* per-group with one group (gs = K) equals per-channel;
* the INT32 product is numpy's int64 matmul, and is unchanged by permuting K;
* with scale_x = scale_w = 1 (integer inputs of magnitude 127 in every row)
  the linear is the plain integer matmul;
* the nibble pack/unpack round trip is exact for all 256 byte values;
* a W4 group whose entries all have the same magnitude maps to +-7;
* the whole linear equals the composition quantize -> product -> dequant.
"""
import numpy as np
import pytest

import oracle
from w8a8_activation_quantized_b200 import synth


@pytest.fixture(scope="module")
def act():
    return synth.activations(64, 512, seed=11, outlier_frac=0.01, outlier_scale=50.0)


def test_code_range_and_argmax(act):
    q, sx = oracle.quantize_act(act)
    assert np.abs(q.astype(np.int32)).max() <= 127
    xa = np.abs(act.astype(np.float32))
    arg = xa.argmax(axis=1)
    picked = q[np.arange(q.shape[0]), arg]
    assert np.all(np.abs(picked.astype(np.int32)) == 127)
    assert np.all(np.sign(picked) == np.sign(act[np.arange(q.shape[0]), arg].astype(np.float32)))
    assert np.all(sx > 0)


@pytest.mark.parametrize("j", [-6, -1, 1, 3])
def test_power_of_two_scaling(act, j):
    x = act[:, :]
    x = x[np.max(np.abs(x.astype(np.float32)), axis=1) * 2.0 ** j < 60000]
    xs = (x.astype(np.float32) * np.float32(2.0 ** j)).astype(np.float16)
    # keep only rows where the scaling stayed exact in fp16 (no underflow)
    exact = np.all(xs.astype(np.float32) == x.astype(np.float32) * np.float32(2.0 ** j), axis=1)
    assert exact.sum() > 10
    q0, s0 = oracle.quantize_act(x[exact])
    q1, s1 = oracle.quantize_act(xs[exact])
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(s1, s0 * np.float32(2.0 ** j))


def test_positive_constant_scaling_away_from_ties(act):
    """q is unchanged for a general positive factor wherever x/scale is not near a .5 tie."""
    c = np.float32(1.37)
    x = act[:16]
    xs = (x.astype(np.float32) * c).astype(np.float16)
    q0, s0 = oracle.quantize_act(x)
    q1, _ = oracle.quantize_act(xs)
    t = x.astype(np.float32) / s0[:, None]
    safe = np.abs(np.abs(t - np.trunc(t)) - 0.5) > 0.05
    np.testing.assert_array_equal(q0[safe], q1[safe])


def test_zero_token():
    x = np.zeros((3, 64), np.float16)
    x[1] = synth.activations(1, 64, seed=3)[0]
    q, sx = oracle.quantize_act(x)
    assert sx[0] == 0 and sx[2] == 0 and sx[1] > 0
    assert not q[0].any() and not q[2].any()
    W = synth.weights(8, 64, seed=3)
    qw, sw = oracle.quantize_weight_pc(W)
    y = oracle.linear_pc(x, qw, sw).view(np.float16)
    assert not y[0].any() and not y[2].any() and y[1].any()


def test_pg_one_group_equals_pc(act):
    W = synth.weights(32, 512, seed=4)
    qw_c, sw_c = oracle.quantize_weight_pc(W)
    qw_g, sw_g = oracle.quantize_weight_pg(W, 512)
    np.testing.assert_array_equal(qw_c, qw_g)
    np.testing.assert_array_equal(sw_c, sw_g[:, 0])
    y_c = oracle.linear_pc(act, qw_c, sw_c)
    y_g = oracle.linear_pg(act, qw_g, sw_g, 512)
    np.testing.assert_array_equal(y_c, y_g)


def test_gemm_is_integer_matmul_and_order_free(act):
    q, _ = oracle.quantize_act(act)
    rng = np.random.default_rng(9)
    w = rng.integers(-128, 128, size=(48, q.shape[1]), dtype=np.int64).astype(np.int8)
    acc = oracle.gemm_i32(q, w)
    ref = q.astype(np.int64) @ w.astype(np.int64).T
    np.testing.assert_array_equal(acc, ref)
    perm = rng.permutation(q.shape[1])
    np.testing.assert_array_equal(oracle.gemm_i32(q[:, perm], w[:, perm]), acc)
    acc_g = oracle.gemm_i32_grouped(q, w, 64)
    np.testing.assert_array_equal(acc_g.astype(np.int64).sum(axis=0), ref)
    np.testing.assert_array_equal(acc_g[3], q[:, 192:256].astype(np.int64) @ w[:, 192:256].astype(np.int64).T)


def test_unit_scales_reduce_to_integer_matmul():
    rng = np.random.default_rng(12)
    M, N, K = 5, 7, 4  # 4 * 127 * 127 < 65504: no fp16 overflow
    xi = rng.integers(-127, 128, size=(M, K))
    xi[:, 0] = 127  # max |x| = 127 in every row -> scale_x = 1
    Wi = rng.integers(-127, 128, size=(N, K))
    Wi[:, 1] = -127  # -> scale_w = 1
    q, sx = oracle.quantize_act(xi.astype(np.float16))
    qw, sw = oracle.quantize_weight_pc(Wi.astype(np.float32))
    assert np.all(sx == 1) and np.all(sw == 1)
    np.testing.assert_array_equal(q, xi)
    y = oracle.linear_pc(xi.astype(np.float16), qw, sw).view(np.float16)
    ref = (xi @ Wi.T).astype(np.float16)  # numpy's own int -> fp16 rounding (nearest even)
    np.testing.assert_array_equal(y, ref)


def test_nibble_round_trip_all_bytes():
    packed = np.arange(256, dtype=np.uint8).reshape(128, 2)
    w = oracle.unpack_int4(packed, 4)
    lo = (np.arange(256) & 15) - 8
    hi = (np.arange(256) >> 4) - 8
    np.testing.assert_array_equal(w.reshape(-1, 2)[:, 0], lo)
    np.testing.assert_array_equal(w.reshape(-1, 2)[:, 1], hi)
    # quantizing integers in [-7, 7] with a group max of 7 returns them unchanged
    # (-8 is never produced: a group holding -8 has max |w| = 8 and scale 8/7)
    W = np.clip(w.astype(np.float32), -7, 7).reshape(64, 8)
    W[:, 0] = 7.0
    packed2, sw = oracle.quantize_weight_int4_pg(W, 8)
    assert np.all(sw == 1.0)
    np.testing.assert_array_equal(oracle.unpack_int4(packed2, 8), W.astype(np.int8))


def test_int4_equal_magnitudes_map_to_seven():
    W = np.float32([[0.3, -0.3, 0.3, 0.3, -0.3, -0.3, 0.3, -0.3]])
    packed, sw = oracle.quantize_weight_int4_pg(W, 8)
    np.testing.assert_array_equal(oracle.unpack_int4(packed, 8)[0], np.sign(W[0]) * 7)


@pytest.mark.parametrize("ydt", [oracle.F16, oracle.BF16])
def test_linear_is_composition(act, ydt):
    W = synth.weights(40, 512, seed=5)
    qw, sw = oracle.quantize_weight_pc(W)
    q, sx = oracle.quantize_act(act)
    y_comp = oracle.dequant_pc(oracle.gemm_i32(q, qw), sx, sw, ydt)
    np.testing.assert_array_equal(oracle.linear_pc(act, qw, sw, ydt=ydt), y_comp)
    qg, sg = oracle.quantize_weight_pg(W, 128)
    y_comp_g = oracle.dequant_pg(oracle.gemm_i32_grouped(q, qg, 128), sx, sg, ydt)
    np.testing.assert_array_equal(oracle.linear_pg(act, qg, sg, 128, ydt=ydt), y_comp_g)
    packed, s4 = oracle.quantize_weight_int4_pg(W, 64)
    w4 = oracle.unpack_int4(packed, 512)
    np.testing.assert_array_equal(oracle.w4a8_linear_pg(act, packed, s4, 64, ydt=ydt),
                                  oracle.linear_pg(act, w4, s4, 64, ydt=ydt))


def test_silu_mul_against_numpy():
    """SiLU(g) * u of the decoder MLP: the oracle's fp64 evaluation rounded once
    equals numpy's own fp64 expression rounded by numpy (nearest even), and
    SiLU's closed-form special values hold."""
    rng = np.random.default_rng(21)
    g = (rng.standard_normal(100_000) * 4).astype(np.float16)
    u = (rng.standard_normal(100_000) * 2).astype(np.float16)
    a = oracle.silu_mul(g, u).view(np.float16)
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    np.testing.assert_array_equal(a, (gd / (1.0 + np.exp(-gd)) * ud).astype(np.float16))
    # silu(0) = 0, silu(g) -> g for large g, silu(g) -> 0 for very negative g
    sp = oracle.silu_mul(np.float16([0.0, 20.0, -30.0]), np.float16([1.0, 1.0, 1.0])).view(np.float16)
    assert sp[0] == 0 and sp[1] == np.float16(20.0) and abs(float(sp[2])) < 1e-6
    # bf16 path: values exact in bf16, checked against torch's rounding of the fp64 result
    import torch
    gb = torch.tensor([0.5, -1.0, 3.0, -7.5], dtype=torch.bfloat16)
    ub = torch.tensor([2.0, 1.5, -0.25, 4.0], dtype=torch.bfloat16)
    got = oracle.silu_mul(gb.view(torch.int16).numpy().view(np.uint16), ub.view(torch.int16).numpy().view(np.uint16),
                          oracle.BF16)
    ref = (gb.double() * torch.sigmoid(gb.double()) * ub.double()).float().to(torch.bfloat16)
    np.testing.assert_array_equal(got, ref.view(torch.int16).numpy().view(np.uint16))
