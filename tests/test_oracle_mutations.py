"""Planted mistakes: each plausible slip in the oracle must fail a pin (CPU only).

A copy of the oracle's C source gets one textual mutation, is compiled into a
temporary library and swapped in; at least one pin of test_oracle_pins.py must
then fail.  The committed oracle itself is never changed.
"""
import ctypes
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_salience as sal

MUTATIONS = {
    "zero_point_sign_in_gemm": ("p += ((int32_t)q[i] - (int32_t)zp) * (int32_t)a[i];",
                                "p += ((int32_t)q[i] + (int32_t)zp) * (int32_t)a[i];"),
    "zero_point_sign_in_quant": ("nearbyintf(-lo / sf)", "nearbyintf(lo / sf)"),
    "activation_scale_group_index": (
        "float scale = oracle_f16_to_f32(s4[n * G + g]) * s_a[m * G + g];",
        "float scale = oracle_f16_to_f32(s4[n * G + g]) * s_a[m * G];"),
    "truncate_instead_of_round": ("float r = nearbyintf(oracle_f16_to_f32(x[i]) / s);",
                                  "float r = truncf(oracle_f16_to_f32(x[i]) / s);"),
    "scale_divisor_128": ("float s = amax / 127.0f;", "float s = amax / 128.0f;"),
    "scale_rounded_to_fp16": ("float s = amax / 127.0f;", "float s = oracle_f16_to_f32(oracle_f32_to_f16(amax / 127.0f));"),
    "scale_as_reciprocal_product": ("float s = amax / 127.0f;", "float s = amax * (1.0f / 127.0f);"),
    "f16_ties_away": ("float r = nearbyintf(units); /* ties to even */",
                      "float r = floorf(units + 0.5f);"),
    "w8_operand_shift": ("p += (int32_t)q[i] * (int32_t)a[i];",
                         "p += (int32_t)q[i] * (int32_t)a[(i + 1) % ORACLE_GROUP];"),
    "activation_row_dropped": (
        "int32_t p = group_partial_w4(A_q + m * K + g * ORACLE_GROUP,",
        "int32_t p = group_partial_w4(A_q + g * ORACLE_GROUP,"),
    "w4_scale_not_rounded_to_fp16": (
        "            float sf = oracle_f16_to_f32(sh);\n            int zi = 0;",
        "            float sf = sc;\n            int zi = 0;"),
    "salience_delta_sign": ("delta[k] = cq - (double)W[n * K + k];", "delta[k] = (double)W[n * K + k] - cq;"),
    "salience_second_order_not_halved": ("acc += fabs(t + 0.5 * t * t);", "acc += fabs(t + t * t);"),
    "salience_no_absolute_value": ("acc += fabs(t + 0.5 * t * t);", "acc += (t + 0.5 * t * t);"),
    "salience_first_group_scale": ("(double)oracle_f16_to_f32(s[n * Gr + g])", "(double)oracle_f16_to_f32(s[n * Gr])"),
    "top_t_ties_high_index_first": ("return i < j ? -1 : (i > j ? 1 : 0);", "return i > j ? -1 : (i < j ? 1 : 0);"),
    "w8_scale_from_wrong_group": ("float v = fabsf(w[i]);\n                if (v > amax) amax = v;\n            }\n            float sc = amax / 127.0f;",
                                  "float v = fabsf(w[i % 64]);\n                if (v > amax) amax = v;\n            }\n            float sc = amax / 127.0f;"),
}


def _pins():
    yield pins.test_f32_to_f16_matches_ieee_rne, ()
    yield pins.test_act_quant_invariants, ()
    yield pins.test_act_quant_ties_half_even_and_zero_group, ()
    yield pins.test_act_quant_scale_keeps_full_precision, ()
    yield pins.test_act_quant_scale_is_correctly_rounded, ()
    yield pins.test_act_quant_lossless_grid, ()
    yield pins.test_w4_invariants, ()
    yield pins.test_w4_lossless_grid_and_special_groups, ()
    yield pins.test_w8_invariants_and_lossless, ()
    for case in pins.CASES:
        yield pins.test_gemm_matches_fp64_brute_force, case
    yield pins.test_group_partials_int64_brute_force, ()
    yield pins.test_partial_bounds_fit_bias_window, ()
    # the global search pins call the module directly (the swapped library)
    for fn in (sal.test_channel_on_the_grid_has_zero_salience, sal.test_zero_gradients_give_zero_salience,
               sal.test_each_group_uses_its_own_scale_and_the_dot_product_spans_the_row,
               sal.test_channels_are_independent, sal.test_top_t_ties_and_bounds, sal.test_top_t_selects_the_largest):
        yield (lambda _o, f=fn: f()), ()
    for eps in (0.25 * sal.S_GRID, -0.375 * sal.S_GRID):
        yield (lambda _o, e=eps: sal.test_one_perturbed_weight_closed_form(e)), ()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path, oracle_mod):
    old, new = MUTATIONS[name]
    with open(oracle._SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(path), "-lm"])
    saved = oracle.lib()
    oracle._lib = oracle.configure(ctypes.CDLL(str(so)))
    try:
        caught = []
        for fn, args in _pins():
            try:
                fn(oracle, *args)
            except AssertionError:
                caught.append(fn.__name__)
        assert caught, f"no pin caught the planted mistake {name}"
    finally:
        oracle._lib = saved
