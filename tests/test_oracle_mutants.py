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
