"""Pins of the oracle for E5M2 operands (the how-to, "Main functions": the FP8 inputs are E4M3
or E5M2), either operand or both: the e5m2 table against the format and torch, exact rational
brute force (decode by formula), identity, the mixed-format transpose symmetry and the format's
extremes.  K-block sums involving e5m2 need up to ~70 bits; the oracle forms them exactly in
128-bit integers, which the extreme-code case exercises."""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_oracle import bf16_exact_rne, e4m3_by_formula, rand_scales


def e5m2_by_formula(code: int) -> Fraction | None:
    """Exact value of a finite e5m2 code, None for infinities and NaN."""
    s = -1 if code & 0x80 else 1
    e = (code >> 2) & 0x1F
    m = code & 3
    if e == 31:
        return None
    if e == 0:
        return s * Fraction(m, 4) * Fraction(1, 2 ** 14)
    return s * (1 + Fraction(m, 4)) * (Fraction(2) ** (e - 15))


FORMULA = {"e4m3": e4m3_by_formula, "e5m2": e5m2_by_formula}


def rand_codes_fmt(rng, shape, fmt):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    if fmt == "e4m3":
        c[(c & 0x7F) == 0x7F] = 0x3C
    else:
        c[((c >> 2) & 0x1F) == 0x1F] = 0x3C  # no infinities or NaN
    return c


def brute(A, fa, sfa, B, fb, sfb, K):
    M, N = A.shape[0], B.shape[0]
    KB = (K + 127) // 128
    da = [FORMULA[fa](c) for c in range(256)]
    db = [FORMULA[fb](c) for c in range(256)]
    out = np.zeros((M, N), dtype=np.uint16)
    for m in range(M):
        for n in range(N):
            total = Fraction(0)
            for kb in range(KB):
                s = Fraction(0)
                for k in range(kb * 128, min(K, kb * 128 + 128)):
                    s += da[A[m, k]] * db[B[n, k]]
                total += s * Fraction(float(sfa[kb, m])) * Fraction(float(sfb[n // 128, kb]))
            out[m, n] = bf16_exact_rne(total)
    return out


def test_e5m2_table_matches_formula_and_torch():
    dec = oracle.e5m2_decode_table()
    tv = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).float().double().numpy()
    for c in range(256):
        v = e5m2_by_formula(c)
        if v is None:
            assert not np.isfinite(dec[c]) and not np.isfinite(tv[c])
            assert np.isinf(dec[c]) == np.isinf(tv[c])
        else:
            assert Fraction(dec[c]) == v and tv[c] == dec[c]


@pytest.mark.parametrize("fa,fb", [("e5m2", "e5m2"), ("e4m3", "e5m2"), ("e5m2", "e4m3")])
@pytest.mark.parametrize("M,N,K,seed", [(3, 4, 32, 1), (2, 130, 160, 2), (4, 3, 300, 3)])
def test_e5m2_brute_force(fa, fb, M, N, K, seed):
    rng = np.random.default_rng(seed)
    KB = (K + 127) // 128
    A, B = rand_codes_fmt(rng, (M, K), fa), rand_codes_fmt(rng, (N, K), fb)
    sfa = rand_scales(rng, (KB, synth.sfa_ld(M)))
    sfb = rand_scales(rng, ((N + 127) // 128, KB))
    np.testing.assert_array_equal(oracle.gemm_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb),
                                  brute(A, fa, sfa, B, fb, sfb, K))


def test_e5m2_extreme_codes_need_more_than_fp64():
    """Largest and smallest magnitudes in one K block: the exact sum spans about 2^-32 .. 2^36."""
    K = 128
    A = np.full((1, K), 0x7B, dtype=np.uint8)          # 57344
    B = np.full((1, K), 0x7B, dtype=np.uint8)
    A[0, 1::2] = 0x01                                   # 2^-16 (smallest subnormal)
    B[0, 1::2] = 0x81                                   # -2^-16
    sfa = np.ones((1, 4), dtype=np.float32)
    sfb = np.ones((1, 1), dtype=np.float32)
    got = oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b="e5m2")
    exact = 64 * Fraction(57344) ** 2 - 64 * Fraction(1, 2 ** 32)
    assert got[0, 0] == bf16_exact_rne(exact)
    np.testing.assert_array_equal(got, brute(A, "e5m2", sfa, B, "e5m2", sfb, K))


def test_e5m2_identity_gives_transpose():
    rng = np.random.default_rng(4)
    K = 256
    A = np.zeros((K, K), dtype=np.uint8)
    A[np.arange(K), np.arange(K)] = 0x3C               # 1.0 in e5m2
    B = rand_codes_fmt(rng, (200, K), "e5m2")
    B[B == 0x80] = 0x00  # -0 contributes like +0: a dot product of zeros is +0
    sfa = np.ones((2, K), dtype=np.float32)
    sfb = np.ones((2, 2), dtype=np.float32)
    C = oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b="e5m2")
    want = torch.from_numpy(B).view(torch.float8_e5m2).float().to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(C, want.T.view(np.uint16))


def test_mixed_formats_transpose_symmetry():
    """With unit scales C(A e4m3, B e5m2) = C(B e5m2, A e4m3)^T exactly: the formats follow the operands."""
    rng = np.random.default_rng(5)
    M, N, K = 12, 20, 384
    A = rand_codes_fmt(rng, (M, K), "e4m3")
    B = rand_codes_fmt(rng, (N, K), "e5m2")
    ones = lambda r, c: np.ones((r, c), dtype=np.float32)  # noqa: E731
    C1 = oracle.gemm_nt(A, ones(3, synth.sfa_ld(M)), B, ones(1, 3), fmt_a="e4m3", fmt_b="e5m2")
    C2 = oracle.gemm_nt(B, ones(3, synth.sfa_ld(N)), A, ones(1, 3), fmt_a="e5m2", fmt_b="e4m3")
    np.testing.assert_array_equal(C1, C2.T)
    C3 = oracle.gemm_nt(A, ones(3, synth.sfa_ld(M)), B, ones(1, 3))  # B read as e4m3: differs
    assert not np.array_equal(C1, C3)
