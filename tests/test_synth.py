"""Checks of the seeded input generator (no GEMM arithmetic here)."""
import numpy as np
import torch

import oracle
import synth


def test_stream_is_counter_based_and_deterministic():
    a = synth.normal_f32(5, 0, 1000)
    b = synth.normal_f32(5, 0, 1000)
    np.testing.assert_array_equal(a, b)
    # any window of the stream equals the same slice of a longer draw
    np.testing.assert_array_equal(synth.normal_f32(5, 101, 50), a[101:151])
    assert not np.array_equal(synth.normal_f32(6, 0, 1000), a)
    big = synth.normal_f32(9, 0, 400000)
    assert abs(big.mean()) < 0.01 and abs(big.std() - 1.0) < 0.01


def test_quantize_1x128_properties():
    x = synth.normal_f32(3, 0, 7 * 300).reshape(7, 300)
    q, sf = synth.quantize_1x128(x)
    assert sf.shape == (3, 8) and q.shape == (7, 300)
    tab = oracle.e4m3_decode_table()
    for r in range(7):
        for kb in range(3):
            blk = slice(kb * 128, min(300, kb * 128 + 128))
            amax = np.abs(x[r, blk]).max()
            assert sf[kb, r] == np.float32(amax) / np.float32(448.0)
            deq = tab[q[r, blk]] * sf[kb, r]
            assert np.max(np.abs(tab[q[r, blk]])) == 448.0      # the block max hits the top code
            assert np.max(np.abs(deq - x[r, blk])) <= amax / 448.0 * 16 + 1e-12


def test_fused_generator_matches_two_step():
    M, K = 5, 384
    rs = synth.row_factors(4, M)
    q1, s1 = synth.quantized_a(8, M, K, row_scale=rs)
    x = synth.normal_f32(8, 0, M * K).reshape(M, K) * rs[:, None]
    q2, s2 = synth.quantize_1x128(x.astype(np.float32))
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s1, s2)
    qb, sb = synth.quantized_b(9, 200, K)
    qb2, sb2 = synth.quantize_128x128(synth.normal_f32(9, 0, 200 * K).reshape(200, K))
    np.testing.assert_array_equal(qb, qb2)
    np.testing.assert_array_equal(sb, sb2)


def test_zero_block_gets_unit_scale():
    x = np.zeros((2, 256), dtype=np.float32)
    x[1, 200] = 3.0
    q, sf = synth.quantize_1x128(x)
    assert sf[0, 0] == 1.0 and sf[1, 0] == 1.0 and sf[0, 1] == 1.0
    assert np.all(q[0] == 0)


def test_row_factors_range_and_masked_counts():
    f = synth.row_factors(2000, 10000)
    assert f.min() >= 1e-2 * 0.999 and f.max() <= 1e2 * 1.001
    lf = np.log10(f)
    assert abs(lf.mean()) < 0.1
    m = synth.masked_counts(5003, 4, 256)
    assert m[0] == 0 and m[3] == 256 and np.all((m >= 0) & (m <= 256))
    assert synth.masked_counts(5000, 1, 1024).tolist() == [1024]


def test_contiguous_layout_padding():
    case = synth.contiguous_case(1, [5, 130, 0, 128], N=16, K=32)
    mi = case["m_indices"]
    assert case["M"] == 128 + 256 + 0 + 128
    assert (mi[:5] == 0).all() and (mi[5:128] == -1).all()
    assert (mi[128:258] == 1).all() and (mi[258:384] == -1).all()
    assert (mi[384:] == 3).all()


def test_e5m2_encoder_matches_torch_in_range():
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.uniform(-57344, 57344, 20000), rng.standard_normal(20000) * 1e-3,
                        rng.standard_normal(20000)]).astype(np.float32)
    mine = np.array([synth.e5m2_encode(x) for x in v], np.uint8)
    ref = torch.from_numpy(v).to(torch.float8_e5m2).view(torch.uint8).numpy()
    np.testing.assert_array_equal(mine, ref)
    assert synth.e5m2_encode(1e9) == 0x7B and synth.e5m2_encode(-1e9) == 0xFB  # saturation at 57344


def test_e5m2_operands_dequantise_close_to_the_draws():
    c = synth.dense_case(3, 8, 130, 256, fmt_a="e5m2", fmt_b="e5m2")
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    a = dec[c["A"]] * np.repeat(c["sfa"][:, :8].T, 128, axis=1)
    assert np.all(np.abs(a).max(axis=1) > 0) and np.isfinite(a).all()
    # the block maximum lands on the largest finite e5m2 value
    assert np.all((c["A"][:, :128] & 0x7F).max(axis=1) == 0x7B)
