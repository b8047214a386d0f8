"""The pins must catch plausible mistakes in the oracle.

Each case copies the oracle's C source, plants one mistake (a dropped term,
a wrong rounding rule, a wrong index or constant), compiles the copy on the
CPU into a temporary directory, swaps it in, and checks that at least one
pin -- the hand-worked golden examples or a brute-force/invariant check --
now fails.  The real oracle is restored afterwards.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle.build import CFLAGS, SRC
from tests import test_oracle_golden as golden_tests
from tests import test_oracle_invariants as inv_tests
from tests import test_oracle_w8a16 as w8a16_tests
from tests import test_oracle_clip as clip_tests
from tests import test_oracle_w4pc as w4pc_tests

MUTATIONS = {
    "round_half_to_even_codes": ("if (fabsf(d) >= 0.5f)", "if (fabsf(d) > 0.5f || (fabsf(d) == 0.5f && fmodf(r, 2.0f) != 0.0f))"),
    "scale_divisor_128": ("float s = amax / 127.0f;\n        sx[m] = s;", "float s = amax / 128.0f;\n        sx[m] = s;"),
    "drop_weight_scale_pc": ("(double)s * (double)sw[n], ydt)", "(double)s, ydt)"),
    "pg_first_group_scale_only": ("sum += (double)a * (double)sw[n * G + g];", "sum += (double)a * (double)sw[n * G];"),
    "int4_nibbles_swapped": ("int nib = (k & 1) ? (b >> 4) : (b & 0x0F);", "int nib = (k & 1) ? (b & 0x0F) : (b >> 4);"),
    "int4_zero_point_7": ("w[n * K + k] = (int8_t)(nib - 8);", "w[n * K + k] = (int8_t)(nib - 7);"),
    "output_ties_away": ("(diff == 0.5 && fmod(fl, 2.0) != 0.0)", "(diff == 0.5)"),
    "product_sign_flip": ("a += (int64_t)qrow[k] * (int64_t)w[n * K + k];\n            if (a > INT32_MAX",
                          "a -= (int64_t)qrow[k] * (int64_t)w[n * K + k];\n            if (a > INT32_MAX"),
    "weight_scale_divisor_128": ("quantize_slab(W + n * K, K, 127.0f,", "quantize_slab(W + n * K, K, 128.0f,"),
    "pg_group_offset_dropped": ("quantize_slab(W + n * K + g * gs, gs,", "quantize_slab(W + n * K, gs,"),
    "w8a16_scale_dropped": ("y[m * N + n] = narrow(a * (double)sw[n], ydt);", "y[m * N + n] = narrow(a, ydt);"),
    "w8a16_weight_sign_dropped": ("a += (double)widen(x, m * K + k, xdt) * (double)w[n * K + k];",
                                  "a += (double)widen(x, m * K + k, xdt) * fabs((double)w[n * K + k]);"),
    "w8a16_pg_first_group_scale_only": ("sum += (double)sw[n * G + g] * part;", "sum += (double)sw[n * G] * part;"),
    "w8a16_pg_group_offset_dropped": ("for (int64_t k = g * gs; k < (g + 1) * gs; ++k)\n                    part +=",
                                      "for (int64_t k = 0; k < gs; ++k)\n                    part +="),
    "clip_interpolation_sign": ("v = a[i] + td;", "v = a[i] - td;"),
    "clip_position_uses_len": ("double pos = p / 100.0 * (double)(len - 1);", "double pos = p / 100.0 * (double)len;"),
    "clip_asymmetric_128": ("clamp_int(oracle_round_half_away(w[k] / s), -127, 127)",
                            "clamp_int(oracle_round_half_away(w[k] / s), -128, 127)"),
    "clip_no_zero_fallback": ("float c = (v == 0.0f) ? amax : v;", "float c = v;"),
    "clip_pg_group_offset_dropped": ("quantize_slab_clip(W + n * K + g * gs, gs,", "quantize_slab_clip(W + n * K, gs,"),
}

PINS = [
    golden_tests.test_pc_worked_example,
    golden_tests.test_pg_worked_example,
    golden_tests.test_w4a8_worked_example,
    lambda _golden: inv_tests.test_nibble_round_trip_all_bytes(),
    lambda _golden: w8a16_tests.test_w8a16_worked_example(),
    lambda _golden: w8a16_tests.test_w8a16_pg_worked_example(),
    lambda _golden: clip_tests.test_clip_pc_worked_example_p90(),
    lambda _golden: clip_tests.test_clip_pc_worked_example_interpolated(),
    lambda _golden: clip_tests.test_clip_pg_worked_example(),
    lambda _golden: clip_tests.test_clip_zero_percentile_falls_back_to_max(),
    lambda _golden: w4pc_tests.test_w4pc_worked_example(),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", *CFLAGS, "-o", str(lib), str(path), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(tmp_path, golden, name):
    old, new = MUTATIONS[name]
    path = _build_mutant(tmp_path, name, old, new)
    saved = oracle._load()
    oracle._lib = oracle._bind(path)
    failures = 0
    try:
        for pin in PINS:
            try:
                pin(golden)
            except (AssertionError, OverflowError):
                failures += 1
    finally:
        oracle._lib = saved
    assert failures > 0, f"no pin caught mutation {name}"
    os.remove(path)


def test_real_oracle_passes_the_same_pins(golden):
    for pin in PINS:
        pin(golden)
