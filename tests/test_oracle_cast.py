"""Pins of the oracle's cast step (BF16 -> e4m3 codes + fine-grained fp32 scales).

The reading (the pages leave the cast to the user): per block (1 x 128 of a row for A,
128 x 128 for B) scale = amax / 448 in fp32 (1 for an all-zero block) and
code = e4m3 round-to-nearest-even of the fp32 quotient x / scale, saturating at 448.
The pins below fix that without restating the oracle's code: exhaustive round trips
of the format, exact ties, the library conversion of torch, properties every correct
quantizer has (the block maximum lands on 448, the RNE error bound, power-of-two
invariance), the scale layouts, and a round trip through the GEMM oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Truncating fp32 -> bf16 bit patterns (the inputs only need to be some bf16 values)."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


DEC = None


def dec():
    global DEC
    if DEC is None:
        DEC = oracle.e4m3_decode_table()
    return DEC


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = dec()[codes].astype(np.float32)
    vals[codes == 0x80] = -0.0
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_encode_ties_to_even_and_neighbours():
    d = dec()
    lo = np.arange(0, 0x7E)
    mid = ((d[lo] + d[lo + 1]) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (d[lo] + d[lo + 1]) / 2)  # exact in fp32
    even = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(oracle.e4m3_encode(mid), even.astype(np.uint8))
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle.e4m3_encode(up), (lo + 1).astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode(down), lo.astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode(-mid), (even | 0x80).astype(np.uint8))


def test_encode_saturates():
    v = np.array([448.0, 449.0, 464.0, 1e30, -500.0, -1e38], dtype=np.float32)
    assert oracle.e4m3_encode(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(-448, 448, 200000), rng.standard_normal(200000) * 1e-2,
                        rng.standard_normal(100000) * 1e-3]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_hand_example_unit_scale():
    row = np.zeros(128, dtype=np.float32)
    row[:4] = [448.0, -224.0, 1.5, 3.375]
    q, sfa = oracle.quantize_rows(f32_to_bf16_bits(row[None]))
    assert sfa.shape == (1, 4) and sfa[0, 0] == 1.0
    # 448 = 1.75 * 2^8, -224 = -1.75 * 2^7, 1.5 = 1.5 * 2^0; between 2 and 4 the spacing is 0.25, so
    # 3.375 is the tie of 3.25 (mantissa 101) and 3.5 (mantissa 110): the even one, 3.5 = 0 1000 110
    assert q[0, :4].tolist() == [0x7E, 0xF6, 0x3C, 0x46]
    assert np.all(q[0, 4:] == 0)


def random_bf16(shape, seed, spread=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    if spread:
        x *= (10.0 ** rng.uniform(-3, 3, shape[:-1] + (1,))).astype(np.float32)
    return f32_to_bf16_bits(x)


@pytest.mark.parametrize("M,K", [(5, 128), (7, 300), (33, 1040)])
def test_rows_block_max_lands_on_448_and_rne_bound(M, K):
    X = random_bf16((M, K), M + K)
    q, sfa = oracle.quantize_rows(X)
    x = bf16_bits_to_f32(X).astype(np.float64)
    d = dec()
    KB = (K + 127) // 128
    for kb in range(KB):
        blk = slice(kb * 128, min(K, kb * 128 + 128))
        s = sfa[kb, :M].astype(np.float64)
        # the element of largest magnitude is coded as +-448
        idx = np.abs(x[:, blk]).argmax(axis=1)
        assert np.all((q[np.arange(M), blk.start + idx] & 0x7F) == 0x7E)
        # RNE: the decoded code is within half a spacing of x / s (plus the fp32 quotient rounding)
        v = x[:, blk] / s[:, None]
        got = d[q[:, blk]]
        e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6)))
        half_spacing = 2.0 ** (e - 3) / 2
        assert np.all(np.abs(got - v) <= half_spacing * (1 + 1e-6) + np.abs(v) * 2.0 ** -23)
        assert np.all(s > 0)


def test_rows_power_of_two_invariance_and_zero_block():
    X = random_bf16((9, 384), 5, spread=False)
    x = bf16_bits_to_f32(X)
    q0, s0 = oracle.quantize_rows(X)
    q1, s1 = oracle.quantize_rows(f32_to_bf16_bits(x * np.float32(2.0 ** 5)))
    assert np.array_equal(q0, q1) and np.array_equal(s1, s0 * np.float32(2.0 ** 5))
    x[3, 128:256] = 0.0
    q2, s2 = oracle.quantize_rows(f32_to_bf16_bits(x))
    assert s2[1, 3] == 1.0 and np.all(q2[3, 128:256] == 0)


def test_rows_scale_layout_column_major_and_grouped():
    X = random_bf16((2, 6, 256), 9)
    q, sfa = oracle.quantize_rows(X)
    assert sfa.shape == (2, 2, 8)  # [G][KB][ld], ld = 6 rounded up to 8
    assert np.all(sfa[:, :, 6:] == 0)  # padding rows are not written
    for g in range(2):
        qg, sg = oracle.quantize_rows(X[g])
        assert np.array_equal(qg, q[g]) and np.array_equal(sg[:, :6], sfa[g, :, :6])
    # row m of K block kb sits at sfa[kb][m]: swapping two rows swaps the scales of that column
    Xs = X[0][[1, 0, 2, 3, 4, 5]]
    _, ss = oracle.quantize_rows(Xs)
    assert np.array_equal(ss[:, [1, 0]], sfa[0][:, :2])


def test_blocks_agree_with_rows_when_row_maxima_agree():
    rng = np.random.default_rng(11)
    x = rng.uniform(-1, 1, (130, 260)).astype(np.float32)
    x[:, 0] = 2.0    # every row of K block 0 has the same maximum
    x[:, 128] = -4.0  # ... and of K block 1
    x[:, 256] = 2.0   # ... and of the partial K block 2
    X = f32_to_bf16_bits(x)
    qr, sr = oracle.quantize_rows(X)
    qb, sb = oracle.quantize_blocks(X)
    assert np.array_equal(qr, qb)
    assert sb.shape == (2, 3)
    for kb in range(3):
        assert np.all(sb[:, kb] == sr[kb, 0])


def test_blocks_max_lands_on_448_per_block():
    X = random_bf16((2, 200, 300), 13, spread=False)
    q, sfb = oracle.quantize_blocks(X)
    x = np.abs(bf16_bits_to_f32(X))
    for g in range(2):
        for nb in range(2):
            for kb in range(3):
                blk = x[g, nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
                i, j = np.unravel_index(blk.argmax(), blk.shape)
                assert (q[g, nb * 128 + i, kb * 128 + j] & 0x7F) == 0x7E
                assert sfb[g, nb, kb] > 0


def test_cast_then_gemm_approximates_the_bf16_product():
    rng = np.random.default_rng(17)
    x = rng.standard_normal((64, 384)).astype(np.float32)
    w = rng.standard_normal((200, 384)).astype(np.float32)
    X, W = f32_to_bf16_bits(x), f32_to_bf16_bits(w)
    A, sfa = oracle.quantize_rows(X)
    B, sfb = oracle.quantize_blocks(W)
    C = bf16_bits_to_f32(oracle.gemm_nt(A, sfa, B, sfb)).astype(np.float64)
    ref = bf16_bits_to_f32(X).astype(np.float64) @ bf16_bits_to_f32(W).astype(np.float64).T
    rel = np.linalg.norm(C - ref) / np.linalg.norm(ref)
    assert rel < 0.05, rel  # e4m3 keeps 3 mantissa bits: a few percent
    # scale semantics: dequantised A = code * scale reproduces x within the e4m3 step
    deq = dec()[A] * np.repeat(sfa[:, :64].T, 128, axis=1)[:, :384]
    assert np.max(np.abs(deq - bf16_bits_to_f32(X))) <= 0.07 * np.abs(bf16_bits_to_f32(X)).max()


# ---------------------------------------------------------------------------- e5m2 target
def dec52():
    return oracle.e5m2_decode_table()


def test_e5m2_encode_round_trips_ties_and_saturation():
    d = dec52()
    codes = np.array([c for c in range(256) if ((c >> 2) & 0x1F) != 0x1F], dtype=np.uint8)
    vals = d[codes].astype(np.float32)
    vals[codes == 0x80] = -0.0
    assert np.array_equal(oracle.e5m2_encode(vals), codes)
    lo = np.arange(0, 0x7B)
    mid = ((d[lo] + d[lo + 1]) / 2).astype(np.float32)
    even = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(oracle.e5m2_encode(mid), even.astype(np.uint8))
    assert np.array_equal(oracle.e5m2_encode(np.nextafter(mid, np.float32(np.inf))), (lo + 1).astype(np.uint8))
    assert oracle.e5m2_encode(np.array([57344, 60000, 1e30, -1e30], np.float32)).tolist() == [0x7B, 0x7B, 0x7B, 0xFB]


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(23)
    v = np.concatenate([rng.uniform(-57344, 57344, 200000), rng.standard_normal(200000) * 1e-3,
                        rng.standard_normal(100000) * 1e-5]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e5m2_encode(v), ref)


def test_e5m2_cast_block_max_and_gemm_round_trip():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((40, 384)).astype(np.float32) * np.float32(1e3)
    w = rng.standard_normal((136, 384)).astype(np.float32)
    X, W = f32_to_bf16_bits(x), f32_to_bf16_bits(w)
    A, sfa = oracle.quantize_rows(X, fmt="e5m2")
    B, sfb = oracle.quantize_blocks(W, fmt="e5m2")
    xa = np.abs(bf16_bits_to_f32(X))
    for kb in range(3):
        idx = xa[:, kb * 128:(kb + 1) * 128].argmax(axis=1)
        assert np.all((A[np.arange(40), kb * 128 + idx] & 0x7F) == 0x7B)  # the maximum lands on 57344
    C = bf16_bits_to_f32(oracle.gemm_nt(A, sfa, B, sfb, fmt_a="e5m2", fmt_b="e5m2")).astype(np.float64)
    ref = bf16_bits_to_f32(X).astype(np.float64) @ bf16_bits_to_f32(W).astype(np.float64).T
    assert np.linalg.norm(C - ref) / np.linalg.norm(ref) < 0.1  # two mantissa bits: ~10% per element
    # with e4m3 the same inputs are closer: the format reaches the codes
    A4, sfa4 = oracle.quantize_rows(X)
    B4, sfb4 = oracle.quantize_blocks(W)
    C4 = bf16_bits_to_f32(oracle.gemm_nt(A4, sfa4, B4, sfb4)).astype(np.float64)
    assert np.linalg.norm(C4 - ref) < np.linalg.norm(C - ref)
