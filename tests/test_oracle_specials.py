"""Pins of the oracle on non-finite input codes (CPU).

The pages say nothing about NaN or infinite inputs; the reading taken is IEEE propagation: a NaN
code makes every output it enters NaN, an infinity gives an infinity with the sign of the product
(scales are positive), infinity times zero and +inf + -inf give NaN.  The expected values below
follow from those rules alone; the finite outputs must equal the product without the special
codes.  e4m3 has NaN codes only (0x7F, 0xFF); e5m2 has +-inf (0x7C, 0xFC) and NaNs (0x7D-0x7F,
0xFD-0xFF).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle

E4M3_ONE, E5M2_ONE = 0x38, 0x3C          # 1.0 in each format
E4M3_MINUS_ONE, E5M2_MINUS_ONE = 0xB8, 0xBC


def is_nan(bits):
    b = np.asarray(bits, dtype=np.uint16)
    return ((b & 0x7F80) == 0x7F80) & ((b & 0x007F) != 0)


def operands(M, N, K, one_a, one_b, seed):
    rng = np.random.default_rng(seed)
    A = np.full((M, K), one_a, dtype=np.uint8)
    B = np.full((N, K), one_b, dtype=np.uint8)
    KB = (K + 127) // 128
    sfa = (rng.random((KB, (M + 3) // 4 * 4)) + 0.5).astype(np.float32)
    sfb = (rng.random(((N + 127) // 128, KB)) + 0.5).astype(np.float32)
    return A, sfa, B, sfb


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e5m2", "e5m2"), ("e4m3", "e5m2"), ("e5m2", "e4m3")])
@pytest.mark.parametrize("nan_code", [0x7F, 0xFF])
def test_nan_code_in_a_poisons_its_row(fa, fb, nan_code):
    M, N, K = 5, 140, 300
    one_a = E4M3_ONE if fa == "e4m3" else E5M2_ONE
    one_b = E4M3_ONE if fb == "e4m3" else E5M2_ONE
    A, sfa, B, sfb = operands(M, N, K, one_a, one_b, 1)
    clean = oracle.gemm_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb)
    A[2, 257] = nan_code  # last, partial K block
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb)
    assert is_nan(C[2]).all()
    keep = np.arange(M) != 2
    np.testing.assert_array_equal(C[keep], clean[keep])


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e5m2", "e5m2")])
def test_nan_code_in_b_poisons_its_column(fa, fb):
    M, N, K = 6, 130, 256
    one_a = E4M3_ONE if fa == "e4m3" else E5M2_ONE
    one_b = E4M3_ONE if fb == "e4m3" else E5M2_ONE
    A, sfa, B, sfb = operands(M, N, K, one_a, one_b, 2)
    clean = oracle.gemm_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb)
    B[129, 3] = 0x7F
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb)
    assert is_nan(C[:, 129]).all()
    np.testing.assert_array_equal(C[:, :129], clean[:, :129])


@pytest.mark.parametrize("fb", ["e5m2", "e4m3"])
def test_e5m2_infinity_keeps_the_sign_of_the_product(fb):
    M, N, K = 3, 4, 128
    one_b = E4M3_ONE if fb == "e4m3" else E5M2_ONE
    minus_b = E4M3_MINUS_ONE if fb == "e4m3" else E5M2_MINUS_ONE
    A, sfa, B, sfb = operands(M, N, K, E5M2_ONE, one_b, 3)
    B[1, :] = minus_b       # column 1: negative products
    B[2, 10] = 0x00         # column 2: the infinity meets a zero -> NaN
    A[0, 10] = 0x7C         # +inf in row 0
    A[1, 10] = 0xFC         # -inf in row 1
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b=fb)
    assert C[0, 0] == 0x7F80 and C[0, 3] == 0x7F80      # +inf * +1
    assert C[0, 1] == 0xFF80                            # +inf * -1
    assert C[1, 0] == 0xFF80 and C[1, 1] == 0x7F80      # -inf * +1, -inf * -1
    assert is_nan(C[0, 2]) and is_nan(C[1, 2])          # inf * 0
    assert not is_nan(C[2]).any() and ((C[2] & 0x7F80) != 0x7F80).all()  # row 2 untouched


def test_opposite_infinities_in_one_sum_give_nan():
    A, sfa, B, sfb = operands(2, 3, 256, E5M2_ONE, E5M2_ONE, 4)
    A[0, 5] = 0x7C    # +inf, first K block
    A[0, 6] = 0xFC    # -inf, same block
    A[1, 5] = 0x7C    # +inf, first block
    A[1, 200] = 0xFC  # -inf, second block: the blocks' sum is +inf + -inf
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b="e5m2")
    assert is_nan(C[0]).all() and is_nan(C[1]).all()


@pytest.mark.parametrize("code", [0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF])
def test_every_e5m2_nan_code_propagates(code):
    A, sfa, B, sfb = operands(1, 2, 128, E5M2_ONE, E5M2_ONE, 5)
    A[0, 0] = code
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b="e5m2")
    assert is_nan(C).all()


def test_grouped_layouts_propagate_the_same_way():
    G, Mmax, N, K = 2, 4, 136, 256
    rng = np.random.default_rng(6)
    A = np.full((G, Mmax, K), E5M2_ONE, dtype=np.uint8)
    B = np.full((G, N, K), E5M2_ONE, dtype=np.uint8)
    sfa = (rng.random((G, 2, 4)) + 0.5).astype(np.float32)
    sfb = (rng.random((G, 2, 2)) + 0.5).astype(np.float32)
    A[1, 0, 7] = 0x7C
    C = oracle.grouped_masked(A, sfa, B, sfb, np.array([4, 4], np.int32), fmt_a="e5m2", fmt_b="e5m2")
    assert (C[1, 0] == 0x7F80).all()
    assert not is_nan(C).any() and ((C[0] & 0x7F80) != 0x7F80).all()
