"""Pin the oracle to the hand-worked examples under tests/golden/.

Each fixture states its sources (page title and section) and the hand
derivation of every number; nothing in them was produced by code here.
"""
import numpy as np
import pytest

import oracle


def _f16(v):
    return np.asarray(v, np.float16)


def test_pc_worked_example(golden):
    g = golden("worked_example_pc_2x4x3.json")
    x = _f16(g["x"])
    q, sx = oracle.quantize_act(x)
    np.testing.assert_array_equal(sx, np.float32(g["scale_x"]))
    np.testing.assert_array_equal(q, np.int8(g["q"]))
    # The fixture's half-to-even alternative must differ: the example separates the two rules.
    assert not np.array_equal(q, np.int8(g["q_if_half_to_even"]))

    qw, sw = oracle.quantize_weight_pc(np.float32(g["W"]))
    np.testing.assert_array_equal(sw, np.float32(g["scale_w"]))
    np.testing.assert_array_equal(qw, np.int8(g["qw"]))

    acc = oracle.gemm_i32(q, qw)
    np.testing.assert_array_equal(acc, np.int32(g["acc"]))

    y = oracle.dequant_pc(acc, sx, sw).view(np.float16)
    np.testing.assert_array_equal(y, _f16(g["y_fp16"]))
    yl = oracle.linear_pc(x, qw, sw).view(np.float16)
    np.testing.assert_array_equal(yl, _f16(g["y_fp16"]))


def test_pg_worked_example(golden):
    g = golden("worked_example_pg_2x4x3_gs2.json")
    gs = g["gs"]
    x = _f16(g["x"])
    q, sx = oracle.quantize_act(x)
    np.testing.assert_array_equal(q, np.int8(g["q"]))
    qw, sw = oracle.quantize_weight_pg(np.float32(g["W"]), gs)
    np.testing.assert_array_equal(sw, np.float32(g["scale_w"]))
    np.testing.assert_array_equal(qw, np.int8(g["qw"]))
    acc_g = oracle.gemm_i32_grouped(q, qw, gs)
    np.testing.assert_array_equal(acc_g, np.int32(g["acc_g"]))
    y = oracle.dequant_pg(acc_g, sx, sw).view(np.float16)
    np.testing.assert_array_equal(y, _f16(g["y_fp16"]))
    yl = oracle.linear_pg(x, qw, sw, gs).view(np.float16)
    np.testing.assert_array_equal(yl, _f16(g["y_fp16"]))
    # y[0][0] is an exact fp16 tie: ties-to-even, not away from zero
    assert float(y[0, 0]) == 157.75


def test_w4a8_worked_example(golden):
    g = golden("worked_example_w4a8_2x4x2_gs2.json")
    gs = g["gs"]
    packed, sw = oracle.quantize_weight_int4_pg(np.float32(g["W"]), gs)
    np.testing.assert_array_equal(packed, np.uint8(g["packed"]))
    np.testing.assert_array_equal(sw, np.float32(g["scale_w"]))
    w = oracle.unpack_int4(packed, 4)
    np.testing.assert_array_equal(w, np.int8(g["qw"]))
    x = _f16(g["x"])
    q, sx = oracle.quantize_act(x)
    acc_g = oracle.gemm_i32_grouped(q, w, gs)
    np.testing.assert_array_equal(acc_g, np.int32(g["acc_g"]))
    y = oracle.w4a8_linear_pg(x, packed, sw, gs).view(np.float16)
    np.testing.assert_array_equal(y, _f16(g["y_fp16"]))


@pytest.mark.parametrize("dt", [oracle.F16, oracle.BF16])
def test_worked_example_in_bf16_input(golden, dt):
    """Every x of the example is exact in bf16 too, so q and scale_x must not change."""
    g = golden("worked_example_pc_2x4x3.json")
    x32 = np.float32(g["x"])
    bits = (x32.view(np.uint32) >> 16).astype(np.uint16) if dt == oracle.BF16 else x32.astype(np.float16)
    q, sx = oracle.quantize_act(bits, dt)
    np.testing.assert_array_equal(q, np.int8(g["q"]))
    np.testing.assert_array_equal(sx, np.float32(g["scale_x"]))
