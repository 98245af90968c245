"""Pins for the CPU oracle: each test checks it against something other than itself.

What pins what (a plausible mistake anywhere in the oracle fails at least one):
  * shape example (news article, GEMM paragraph) with hand-computed values  -> layout/transposition, scale use
  * exact rational brute force, decode by formula, exact bf16 rounding     -> dropped terms, K-block edges,
                                                                              wrong sfa/sfb index (N > 128, partial K)
  * e4m3 table vs the format formula and vs torch.float8_e4m3fn             -> decode table
  * identity / permutation operands                                        -> operand order, row/col indexing
  * power-of-two rescaling of sfa and sfb                                  -> scale placement
  * grouped == per-group dense, padding / masked rows untouched            -> group routing
  * fp64 -> bf16 against an integer-bit implementation and torch           -> output rounding
"""
from __future__ import annotations

import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# independent helpers written from the number formats (no oracle code)
# ---------------------------------------------------------------------------
def e4m3_by_formula(code: int) -> Fraction | None:
    """Exact value of an e4m3fn code, None for NaN."""
    s = -1 if code & 0x80 else 1
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 15 and m == 7:
        return None
    if e == 0:
        return s * Fraction(m, 8) * Fraction(1, 64)
    return s * (1 + Fraction(m, 8)) * (Fraction(2) ** (e - 7))


def bf16_exact_rne(x: Fraction) -> int:
    """bf16 bit pattern of the exact rational x rounded once, to nearest even."""
    if x == 0:
        return 0
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    # now 2^e <= a < 2^(e+1)
    q = max(e - 7, -133)
    r = a / (Fraction(2) ** q)
    fl = r.numerator // r.denominator
    rem = r - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    y = fl * (Fraction(2) ** q)
    if y >= Fraction(2) ** 128:
        return sign | 0x7F80
    bits = struct.unpack("<I", struct.pack("<f", float(y)))[0]
    assert Fraction(float(y)) == y
    return sign | (bits >> 16)


def brute_force(A, sfa, B, sfb, K):
    """Exact rational C[m,n] with decode by formula, then one exact RNE to bf16."""
    M, N = A.shape[0], B.shape[0]
    KB = (K + 127) // 128
    dec = [e4m3_by_formula(c) for c in range(256)]
    out = np.zeros((M, N), dtype=np.uint16)
    for m in range(M):
        for n in range(N):
            total = Fraction(0)
            for kb in range(KB):
                s = Fraction(0)
                for k in range(kb * 128, min(K, kb * 128 + 128)):
                    s += dec[A[m, k]] * dec[B[n, k]]
                total += s * Fraction(float(sfa[kb, m])) * Fraction(float(sfb[n // 128, kb]))
            out[m, n] = bf16_exact_rne(total)
    return out


def rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return c


def rand_scales(rng, shape):
    return (2.0 ** rng.uniform(-12, 4, size=shape) * rng.uniform(1, 2, size=shape)).astype(np.float32)


def f32(bits):
    return oracle.bf16_bits_to_f32(bits)


# ---------------------------------------------------------------------------
# golden: the pages' 3x2 . 2x4 -> 3x4 shape example
# ---------------------------------------------------------------------------
def _read_golden(name):
    blocks, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.replace("_", "").isalpha():
                cur = line
                blocks[cur] = []
            else:
                blocks[cur].append([float(v) for v in line.split()])
    return {k: np.array(v) for k, v in blocks.items()}


def test_shape_example_golden():
    g = _read_golden("shape_example_3x2x4.txt")
    A = np.array([[synth.e4m3_encode(v) for v in row] for row in g["A"]], dtype=np.uint8)
    Bt = np.array([[synth.e4m3_encode(v) for v in row] for row in g["B"].T], dtype=np.uint8)
    assert A.shape == (3, 2) and Bt.shape == (4, 2)
    ones_a = np.ones((1, 4), dtype=np.float32)
    ones_b = np.ones((1, 1), dtype=np.float32)
    C = oracle.gemm_nt(A, ones_a, Bt, ones_b)
    assert C.shape == (3, 4)
    np.testing.assert_array_equal(f32(C), g["C"].astype(np.float32))
    sfa = np.zeros((1, 4), dtype=np.float32)
    sfa[0, :3] = g["SFA"][0]
    sfb = g["SFB"].astype(np.float32).reshape(1, 1)
    Cs = oracle.gemm_nt(A, sfa, Bt, sfb)
    np.testing.assert_array_equal(f32(Cs), g["C_SCALED"].astype(np.float32))


# ---------------------------------------------------------------------------
# brute force, exact rationals
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 1, 0), (3, 4, 2, 1), (5, 5, 128, 2), (4, 3, 129, 3),
                                        (2, 5, 300, 4), (3, 2, 256, 5)])
def test_brute_force_small(M, N, K, seed):
    rng = np.random.default_rng(seed)
    KB = (K + 127) // 128
    A, B = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    ld = synth.sfa_ld(M)
    sfa = rand_scales(rng, (KB, ld))
    sfb = rand_scales(rng, ((N + 127) // 128, KB))
    np.testing.assert_array_equal(oracle.gemm_nt(A, sfa, B, sfb), brute_force(A, sfa, B, sfb, K))


def test_brute_force_sfb_blocks():
    """N spans two 128-row blocks of B and K ends in a partial block."""
    rng = np.random.default_rng(11)
    M, N, K = 2, 133, 300
    A, B = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = rand_scales(rng, (3, 4))
    sfb = rand_scales(rng, (2, 3))
    np.testing.assert_array_equal(oracle.gemm_nt(A, sfa, B, sfb), brute_force(A, sfa, B, sfb, K))


def test_brute_force_extremes():
    """Largest magnitudes (448) and smallest subnormals (2^-9) in one product."""
    M, N, K = 2, 2, 130
    A = np.full((M, K), 0x7E, dtype=np.uint8)
    A[1] = 0x01
    A[1, 128:] = 0xFE
    B = np.full((N, K), 0x7E, dtype=np.uint8)
    B[1, ::2] = 0x81
    sfa = np.array([[1.0, 2.0 ** -20, 0, 0], [3.0, 0.75, 0, 0]], dtype=np.float32)
    sfb = np.array([[1.5, 2.0 ** -7]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.gemm_nt(A, sfa, B, sfb), brute_force(A, sfa, B, sfb, K))


# ---------------------------------------------------------------------------
# e4m3 decode and encode
# ---------------------------------------------------------------------------
def test_decode_table_matches_formula_and_torch():
    tab = oracle.e4m3_decode_table()
    ref_torch = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = e4m3_by_formula(c)
        if v is None:
            assert math.isnan(tab[c]) and math.isnan(ref_torch[c])
        else:
            assert tab[c] == float(v) == ref_torch[c], c
    assert np.nanmax(tab) == 448.0 and np.nanmin(tab) == -448.0
    assert tab[1] == 2.0 ** -9


def test_encode_roundtrip_and_rne():
    tab = oracle.e4m3_decode_table()
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert synth.e4m3_encode(tab[c]) == c, hex(c)
    # midpoints between neighbouring positive codes round to the even code
    pos = [tab[c] for c in range(0x7F)]
    for c in range(0x7E):
        mid = (pos[c] + pos[c + 1]) / 2
        if float(np.float32(mid)) != mid:
            continue
        expect = c if c % 2 == 0 else c + 1
        assert synth.e4m3_encode(mid) == expect, (c, mid)
        assert synth.e4m3_encode(-mid) == 0x80 | expect
    assert synth.e4m3_encode(1000.0) == 0x7E and synth.e4m3_encode(-1e30) == 0xFE
    assert synth.e4m3_encode(2.0 ** -11) == 0x00  # below half the smallest subnormal
    # the encoder agrees with torch's own fp32 -> e4m3fn conversion (inside the finite range)
    x = synth.normal_f32(77, 0, 20000) * np.float32(100.0)
    x = np.clip(x, -448, 448).astype(np.float32)
    ours = np.array([synth.e4m3_encode(v) for v in x], dtype=np.uint8)
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, theirs)


# ---------------------------------------------------------------------------
# structural special cases
# ---------------------------------------------------------------------------
ONE = 0x38  # e4m3 code of 1.0


def test_identity_gives_transpose():
    rng = np.random.default_rng(5)
    n = 160
    A = np.zeros((n, n), dtype=np.uint8)
    A[np.arange(n), np.arange(n)] = ONE
    B = rand_codes(rng, (96, n))
    sfa = np.ones((2, n), dtype=np.float32)
    sfb = np.ones((1, 2), dtype=np.float32)
    C = oracle.gemm_nt(A, sfa, B, sfb)
    tab = oracle.e4m3_decode_table()
    # e4m3 values are exact in bf16, so C == B^T exactly
    np.testing.assert_array_equal(f32(C), tab[B.T].astype(np.float32))


def test_permutation_rows():
    rng = np.random.default_rng(6)
    M, N, K = 70, 140, 256
    A, B = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = rand_scales(rng, (2, synth.sfa_ld(M)))
    sfb = rand_scales(rng, (2, 2))
    perm = rng.permutation(M)
    sfa_p = np.zeros_like(sfa)
    sfa_p[:, :M] = sfa[:, perm]
    C = oracle.gemm_nt(A, sfa, B, sfb)
    Cp = oracle.gemm_nt(A[perm], sfa_p, B, sfb)
    np.testing.assert_array_equal(Cp, C[perm])
    # a permutation matrix as the LHS selects columns of B: C[m, n] = B[n, q[m]]
    P = np.zeros((K, K), dtype=np.uint8)
    q = rng.permutation(K)
    P[np.arange(K), q] = ONE
    CB = oracle.gemm_nt(P, np.ones((2, K), np.float32), B, np.ones((2, 2), np.float32))
    tab = oracle.e4m3_decode_table()
    np.testing.assert_array_equal(f32(CB), tab[B[:, q].T].astype(np.float32))


def test_power_of_two_rescaling():
    rng = np.random.default_rng(7)
    M, N, K = 9, 200, 384
    A, B = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = rand_scales(rng, (3, synth.sfa_ld(M)))
    sfb = rand_scales(rng, (2, 3))
    C = oracle.gemm_nt(A, sfa, B, sfb)
    for j, i in [(3, 0), (0, 5), (4, 9), (-6, -2)]:
        C2 = oracle.gemm_nt(A, sfa * np.float32(2.0 ** j), B, sfb * np.float32(2.0 ** -i))
        np.testing.assert_array_equal(f32(C2), f32(C) * np.float32(2.0 ** (j - i)))


def test_zero_scale_block_contributes_nothing():
    rng = np.random.default_rng(8)
    M, N, K = 4, 6, 384
    A, B = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = rand_scales(rng, (3, 4))
    sfb = rand_scales(rng, (1, 3))
    sfa0 = sfa.copy()
    sfa0[1, :] = 0.0
    A0 = A.copy()
    A0[:, 128:256] = 0
    np.testing.assert_array_equal(oracle.gemm_nt(A, sfa0, B, sfb), oracle.gemm_nt(A0, sfa, B, sfb))


# ---------------------------------------------------------------------------
# grouped layouts
# ---------------------------------------------------------------------------
def test_contiguous_equals_per_group_dense():
    case = synth.contiguous_case(21, [100, 0, 300, 37], N=136, K=384)
    A, sfa, B, sfb, mi = case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"]
    canary = np.full((case["M"], case["N"]), 0xFFFF, dtype=np.uint16)
    C = oracle.grouped_contiguous(A, sfa, B, sfb, mi, C=canary)
    for g in range(case["G"]):
        rows = np.nonzero(mi == g)[0]
        if rows.size == 0:
            continue
        sub_sfa = np.zeros((sfa.shape[0], synth.sfa_ld(rows.size)), np.float32)
        sub_sfa[:, :rows.size] = sfa[:, rows]
        ref = oracle.gemm_nt(A[rows], sub_sfa, B[g], sfb[g])
        np.testing.assert_array_equal(C[rows], ref)
    pad = mi < 0
    assert pad.sum() == case["M"] - sum(case["group_rows"])
    assert np.all(C[pad] == 0xFFFF)
    # a row subset gives the same rows
    pick = np.array([0, 5, 99, 384, 500, 520], dtype=np.int32)
    sub = oracle.grouped_contiguous(A, sfa, B, sfb, mi, rows=pick)
    live = mi[pick] >= 0
    np.testing.assert_array_equal(sub[live], C[pick][live])


def test_masked_equals_per_group_dense_and_untouched():
    case = synth.masked_case(22, G=4, Mmax=160, N=144, K=256, masked_m=[0, 37, 160, 129])
    A, sfa, B, sfb, mm = case["A"], case["sfa"], case["B"], case["sfb"], case["masked_m"]
    canary = np.full((4, 160, 144), 0xFFFF, dtype=np.uint16)
    C = oracle.grouped_masked(A, sfa, B, sfb, mm, C=canary)
    for g in range(4):
        v = int(mm[g])
        if v:
            ref = oracle.gemm_nt(A[g, :v], sfa[g], B[g], sfb[g])
            np.testing.assert_array_equal(C[g, :v], ref)
        assert np.all(C[g, v:] == 0xFFFF)


def test_dense_rows_subset():
    case = synth.dense_case(23, 40, 136, 256)
    full = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    rows = np.array([39, 0, 17, 17], dtype=np.int32)
    sub = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], rows=rows)
    np.testing.assert_array_equal(sub, full[rows])


# ---------------------------------------------------------------------------
# fp64 -> bf16 rounding
# ---------------------------------------------------------------------------
def bf16_by_bits(x: np.ndarray) -> np.ndarray:
    """Integer-bit RNE of fp64 to bf16 (normal range), an independent implementation."""
    b = x.view(np.uint64)
    sign = ((b >> np.uint64(63)) << np.uint64(15)).astype(np.uint32)
    exp = ((b >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    man = b & np.uint64((1 << 52) - 1)
    keep = man >> np.uint64(45)                   # top 7 mantissa bits
    rest = man & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rest > half) | ((rest == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    val = ((exp - 1023 + 127).astype(np.uint64) << np.uint64(7)) + keep + up.astype(np.uint64)
    return (sign | val.astype(np.uint32)).astype(np.uint16)


def test_bf16_rounding_crafted():
    one = 1.0
    ulp = 2.0 ** -7
    assert oracle.bf16_from_f64(one + ulp / 2) == 0x3F80            # tie -> even (down)
    assert oracle.bf16_from_f64(one + 3 * ulp / 2) == 0x3F82        # tie -> even (up)
    assert oracle.bf16_from_f64(one + ulp / 2 + 2.0 ** -40) == 0x3F81   # just above the tie
    assert oracle.bf16_from_f64(one + ulp / 2 - 2.0 ** -40) == 0x3F80   # just below the tie
    # a value whose fp32 rounding lands exactly on a bf16 tie: double rounding would go wrong
    x = one + ulp / 2 + 2.0 ** -30
    assert float(np.float32(x)) == one + ulp / 2
    assert oracle.bf16_from_f64(x) == 0x3F81
    assert oracle.bf16_from_f64(-2.5) == 0xC020
    assert oracle.bf16_from_f64(0.0) == 0 and oracle.bf16_from_f64(-0.0) == 0x8000
    assert oracle.bf16_from_f64(3.4e38) == 0x7F80                   # rounds past the largest finite
    assert oracle.bf16_from_f64(3.38e38) == 0x7F7E
    assert oracle.bf16_from_f64(float("inf")) == 0x7F80
    assert oracle.bf16_from_f64(float("nan")) & 0x7FC0 == 0x7FC0
    assert oracle.bf16_from_f64(2.0 ** -133) == 0x0001              # smallest bf16 subnormal
    assert oracle.bf16_from_f64(2.0 ** -134) == 0x0000              # tie -> even (zero)
    assert oracle.bf16_from_f64(3 * 2.0 ** -134) == 0x0002          # tie -> even (up)


def test_bf16_rounding_random_vs_bits_and_torch():
    rng = np.random.default_rng(9)
    x = rng.standard_normal(200000) * np.exp2(rng.uniform(-60, 60, 200000))
    # plant exact ties and near-ties
    x[:1000] = np.float64(1.0 + 2.0 ** -8) * np.exp2(rng.integers(-50, 50, 1000))
    ours = np.array([oracle.bf16_from_f64(v) for v in x], dtype=np.uint16)
    np.testing.assert_array_equal(ours, bf16_by_bits(x))
    x32 = x.astype(np.float32).astype(np.float64)   # fp32-exact values: torch's fp32->bf16 must agree
    ours32 = np.array([oracle.bf16_from_f64(v) for v in x32[:50000]], dtype=np.uint16)
    theirs = torch.from_numpy(x32[:50000].astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours32, theirs)
