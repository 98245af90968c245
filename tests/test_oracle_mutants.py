"""The oracle's pins catch plausible mistakes.

Each case compiles a copy of the oracle with one planted mistake (on the CPU, in a
temporary directory), points the oracle module at it and checks that at least one
pin of tests/test_oracle.py fails.  The real oracle is restored afterwards.
"""
from __future__ import annotations

import pathlib
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = pathlib.Path(oracle.__file__).with_name("fp8gemm_oracle.c")

MUTANTS = {
    # wrong block of B scales: ignores the 128-row block of n
    "sfb_index": ("(size_t)(n / ORC_BLOCK) * KB + kb", "(size_t)kb"),
    # the last, partial K block is dropped
    "drop_partial_k": ("int k1 = k0 + ORC_BLOCK < K ? k0 + ORC_BLOCK : K;",
                       "int k1 = k0 + ORC_BLOCK <= K ? k0 + ORC_BLOCK : k0;"),
    # A scales read row-major instead of column-major
    "sfa_layout": ("sfa_m[(size_t)kb * ld]", "sfa_m[(size_t)kb]"),
    # output rounded through fp32 first (double rounding)
    "double_rounding": ("double r = nearbyint(scaled);",
                        "double r = nearbyint(ldexp((double)(float)x, -q));"),
    # an operand indexed transposed
    "transposed_b": ("dec[a_row[k]] * dec[b_row[k]]",
                     "dec[a_row[k]] * dec[B[(size_t)(k % N) * K + (n % K)]]"),
    # a sign error in the decode table
    "decode_sign": ("g_dec[code] = sign ? -v : v;", "g_dec[code] = v;"),
    # scales applied once per element instead of per K block (last block's scale for all)
    "scale_once": ("acc += s * scale;", "acc = (acc + s) * 1.0; (void)scale; if (kb == KB - 1) acc *= scale;"),
}

PINS = [
    pins.test_shape_example_golden,
    lambda: [pins.test_brute_force_small(*p) for p in [(3, 4, 2, 1), (4, 3, 129, 3), (2, 5, 300, 4)]],
    pins.test_brute_force_sfb_blocks,
    pins.test_brute_force_extremes,
    pins.test_decode_table_matches_formula_and_torch,
    pins.test_identity_gives_transpose,
    pins.test_permutation_rows,
    pins.test_power_of_two_rescaling,
    pins.test_bf16_rounding_crafted,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTANTS[name]
    text = SRC.read_text()
    assert text.count(before) == 1, name
    (tmp_path / "m.c").write_text(text.replace(before, after))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", str(tmp_path / "m.c"), "-o", str(so), "-lm"])
    saved = oracle._lib()
    oracle._LIB = oracle.load(so)
    caught = []
    try:
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "brute_force_small"))
    finally:
        oracle._LIB = saved
    assert caught, f"no pin caught the planted mistake {name!r}"


# ---------------------------------------------------------------------------- the cast step
from tests import test_oracle_cast as cast_pins  # noqa: E402

CAST_MUTANTS = {
    # ties rounded away from zero instead of to even (e4m3, e5m2)
    "cast_ties_away": ("else c = (lo % 2 == 0) ? lo : hi;", "else c = hi;"),
    "cast_ties_away_e5m2": ("else c = (lo & 1) ? hi : lo;", "else c = hi;"),
    # the inverse scale
    "cast_inverse_scale": ("volatile float s = fmt == 0 ? amax / 448.0f : amax / 57344.0f;",
                           "volatile float s = fmt == 0 ? 448.0f / amax : 57344.0f / amax;"),
    # non-saturating conversion: magnitudes above 448 become NaN
    "cast_no_saturation": ("if (a >= dec[0x7E]) return sign | 0x7E;",
                           "if (a > dec[0x7E]) return sign | 0x7F; if (a == dec[0x7E]) return sign | 0x7E;"),
    # A scales stored row-major
    "cast_sfa_row_major": ("sfa[((size_t)g * KB + kb) * ld + m] = s;", "sfa[((size_t)g * M + m) * KB + kb] = s;"),
    # block maximum taken over the first row of the block only
    "cast_block_amax_first_row": ("float a = fabsf(bf16_to_f32(x[(size_t)n * K + k]));",
                                  "float a = (n == n0) ? fabsf(bf16_to_f32(x[(size_t)n * K + k])) : 0.0f;"),
}

CAST_PINS = [
    cast_pins.test_encode_round_trips_every_finite_code,
    cast_pins.test_encode_ties_to_even_and_neighbours,
    cast_pins.test_encode_saturates,
    cast_pins.test_encode_matches_torch_in_range,
    cast_pins.test_hand_example_unit_scale,
    lambda: cast_pins.test_rows_block_max_lands_on_448_and_rne_bound(7, 300),
    cast_pins.test_rows_power_of_two_invariance_and_zero_block,
    cast_pins.test_rows_scale_layout_column_major_and_grouped,
    cast_pins.test_blocks_agree_with_rows_when_row_maxima_agree,
    cast_pins.test_blocks_max_lands_on_448_per_block,
    cast_pins.test_cast_then_gemm_approximates_the_bf16_product,
    cast_pins.test_e5m2_encode_round_trips_ties_and_saturation,
    cast_pins.test_e5m2_encode_matches_torch_in_range,
    cast_pins.test_e5m2_cast_block_max_and_gemm_round_trip,
]


@pytest.mark.parametrize("name", sorted(CAST_MUTANTS))
def test_cast_pins_catch_planted_mistake(name, tmp_path):
    before, after = CAST_MUTANTS[name]
    text = SRC.read_text()
    assert text.count(before) == 1, name
    (tmp_path / "m.c").write_text(text.replace(before, after))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", str(tmp_path / "m.c"), "-o", str(so), "-lm"])
    saved = oracle._lib()
    oracle._LIB = oracle.load(so)
    caught = []
    try:
        for pin in CAST_PINS:
            try:
                pin()
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(getattr(pin, "__name__", "rows_block_max"))
    finally:
        oracle._LIB = saved
    assert caught, f"no pin caught the planted mistake {name!r}"


# ---------------------------------------------------------------------------- e5m2 operands
from tests import test_oracle_e5m2 as e5m2_pins  # noqa: E402

E5M2_MUTANTS = {
    # exponent bias 16 instead of 15
    "e5m2_bias": ("v = ldexp(1.0 + (double)m / 4.0, e - 15);", "v = ldexp(1.0 + (double)m / 4.0, e - 16);"),
    # integer units of e5m2 off by one binade
    "e5m2_quantum": ("return fmt == 0 ? 9 : 16;", "return fmt == 0 ? 9 : 15;"),
    # the two operands' formats swapped
    "e5m2_swapped": ("ua[c] = code_units(fa, (uint8_t)c); ub[c] = code_units(fb, (uint8_t)c);",
                     "ua[c] = code_units(fb, (uint8_t)c); ub[c] = code_units(fa, (uint8_t)c);"),
}

E5M2_PINS = [
    e5m2_pins.test_e5m2_table_matches_formula_and_torch,
    lambda: [e5m2_pins.test_e5m2_brute_force(fa, fb, 3, 4, 32, 1)
             for fa, fb in [("e5m2", "e5m2"), ("e4m3", "e5m2"), ("e5m2", "e4m3")]],
    e5m2_pins.test_e5m2_extreme_codes_need_more_than_fp64,
    e5m2_pins.test_e5m2_identity_gives_transpose,
    e5m2_pins.test_mixed_formats_transpose_symmetry,
]


@pytest.mark.parametrize("name", sorted(E5M2_MUTANTS))
def test_e5m2_pins_catch_planted_mistake(name, tmp_path):
    before, after = E5M2_MUTANTS[name]
    text = SRC.read_text()
    assert text.count(before) == 1, name
    (tmp_path / "m.c").write_text(text.replace(before, after))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", str(tmp_path / "m.c"), "-o", str(so), "-lm"])
    saved = oracle._lib()
    oracle._LIB = oracle.load(so)
    caught = []
    try:
        for pin in E5M2_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "brute_force"))
    finally:
        oracle._LIB = saved
    assert caught, f"no pin caught the planted mistake {name!r}"


# ---------------------------------------------------------------------------- non-finite codes
from tests import test_oracle_specials as special_pins  # noqa: E402

SPECIAL_MUTANTS = {
    # non-finite codes counted as zero in the exact integer sums
    "specials_dropped": ("special = !isfinite(deca[a_row[k]]) || !isfinite(decb[b_row[k]]);", "special = 0;"),
    # a special block summed with the finite codes only
    "specials_skipped": ("for (int k = k0; k < k1; ++k) s += deca[a_row[k]] * decb[b_row[k]];",
                         "for (int k = k0; k < k1; ++k) if (isfinite(deca[a_row[k]] * decb[b_row[k]])) "
                         "s += deca[a_row[k]] * decb[b_row[k]];"),
}

SPECIAL_PINS = [
    lambda: [special_pins.test_nan_code_in_a_poisons_its_row(fa, fb, 0x7F)
             for fa, fb in [("e5m2", "e5m2"), ("e4m3", "e5m2")]],
    lambda: special_pins.test_e5m2_infinity_keeps_the_sign_of_the_product("e5m2"),
    special_pins.test_opposite_infinities_in_one_sum_give_nan,
    lambda: special_pins.test_every_e5m2_nan_code_propagates(0x7E),
]


@pytest.mark.parametrize("name", sorted(SPECIAL_MUTANTS))
def test_special_pins_catch_planted_mistake(name, tmp_path):
    before, after = SPECIAL_MUTANTS[name]
    text = SRC.read_text()
    assert text.count(before) == 1, name
    (tmp_path / "m.c").write_text(text.replace(before, after))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", str(tmp_path / "m.c"), "-o", str(so), "-lm"])
    saved = oracle._lib()
    oracle._LIB = oracle.load(so)
    caught = 0
    try:
        for pin in SPECIAL_PINS:
            try:
                pin()
            except AssertionError:
                caught += 1
    finally:
        oracle._LIB = saved
    assert caught, f"no pin caught the planted mistake {name!r}"
