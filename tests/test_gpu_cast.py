"""GPU parity of the cast step (BF16 -> e4m3 codes + fp32 scales) against the oracle: codes and
scales are byte work and must be bit-identical.  Shapes span several blocks with ragged tails,
padding rows of the column-major scale layout, groups, all-zero blocks and extreme magnitudes,
plus full-size activation and weight shapes of the benchmark; the last test casts and multiplies
on the GPU and checks the product against the oracle's cast and GEMM."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import bits_of, close

pytestmark = pytest.mark.gpu


def bf16_inputs(shape, seed, spread=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if spread:  # row magnitudes over six decades
        x = x * torch.pow(10.0, torch.empty(shape[:-1] + (1,)).uniform_(-3, 3, generator=g))
    return x.to(torch.bfloat16)


def as_bits(x: torch.Tensor) -> np.ndarray:
    return x.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    return lib


@pytest.mark.parametrize("shape", [(1, 16), (5, 128), (7, 272), (33, 1040), (3, 6, 384), (129, 256)])
def test_cast_rows_bit_exact(fg, shape):
    x = bf16_inputs(shape, sum(shape))
    q, sfa = fg.cast_fp8_rows(x.cuda())
    torch.cuda.synchronize()
    q_ref, sfa_ref = oracle.quantize_rows(as_bits(x))
    M = shape[-2]
    assert np.array_equal(q.cpu().numpy(), q_ref)
    got = sfa.cpu().numpy()
    assert np.array_equal(got[..., :M].view(np.uint32), sfa_ref[..., :M].view(np.uint32))
    assert np.all(got[..., M:] == 0)  # padding rows of the scale columns are not written


@pytest.mark.parametrize("shape", [(8, 16), (130, 272), (300, 1040), (2, 129, 384)])
def test_cast_blocks_bit_exact(fg, shape):
    w = bf16_inputs(shape, 7 * sum(shape), spread=False)
    q, sfb = fg.cast_fp8_blocks(w.cuda())
    torch.cuda.synchronize()
    q_ref, sfb_ref = oracle.quantize_blocks(as_bits(w))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sfb.cpu().numpy().view(np.uint32), sfb_ref.view(np.uint32))


def test_cast_zero_blocks_and_extremes(fg):
    x = bf16_inputs((4, 512), 3, spread=False).float()
    x[1, 128:256] = 0.0                      # all-zero block: scale 1, codes 0
    x[2, :128] = torch.finfo(torch.bfloat16).max  # largest bf16
    x[2, 1] = -x[2, 1]
    x[3, 256:384] = 2.0 ** -130              # subnormal bf16 inputs
    x = x.to(torch.bfloat16)
    for cast, ref in ((fg.cast_fp8_rows, oracle.quantize_rows), (fg.cast_fp8_blocks, oracle.quantize_blocks)):
        q, s = cast(x.cuda())
        torch.cuda.synchronize()
        q_ref, s_ref = ref(as_bits(x))
        assert np.array_equal(q.cpu().numpy(), q_ref)
        got = s.cpu().numpy()
        sl = (slice(None), slice(0, 4)) if cast is fg.cast_fp8_rows else (slice(None), slice(None))
        assert np.array_equal(got[sl].view(np.uint32), s_ref[sl].view(np.uint32))


@pytest.mark.parametrize("M,N,K", [(4096, 2112, 7168), (128, 7168, 16384)])
def test_cast_full_size(fg, M, N, K):
    x = bf16_inputs((M, K), M + K)
    w = bf16_inputs((N, K), N + K, spread=False)
    qa, sfa = fg.cast_fp8_rows(x.cuda())
    qb, sfb = fg.cast_fp8_blocks(w.cuda())
    torch.cuda.synchronize()
    qa_ref, sfa_ref = oracle.quantize_rows(as_bits(x))
    qb_ref, sfb_ref = oracle.quantize_blocks(as_bits(w))
    assert np.array_equal(qa.cpu().numpy(), qa_ref)
    assert np.array_equal(sfa.cpu().numpy()[:, :M].view(np.uint32), sfa_ref[:, :M].view(np.uint32))
    assert np.array_equal(qb.cpu().numpy(), qb_ref)
    assert np.array_equal(sfb.cpu().numpy().view(np.uint32), sfb_ref.view(np.uint32))


def test_cast_then_gemm_on_gpu(fg):
    M, N, K = 300, 520, 1152
    x = bf16_inputs((M, K), 21)
    w = bf16_inputs((N, K), 22, spread=False)
    qa, sfa = fg.cast_fp8_rows(x.cuda())
    qb, sfb = fg.cast_fp8_blocks(w.cuda())
    C = fg.gemm_fp8_fp8_bf16_nt(qa, sfa, qb, sfb)
    torch.cuda.synchronize()
    qa_ref, sfa_ref = oracle.quantize_rows(as_bits(x))
    qb_ref, sfb_ref = oracle.quantize_blocks(as_bits(w))
    close(bits_of(C), oracle.gemm_nt(qa_ref, sfa_ref, qb_ref, sfb_ref), "cast + gemm")


@pytest.mark.parametrize("s", [1.5, 1.25, 1.75, 0.75])
def test_cast_quotients_exactly_on_e4m3_midpoints(fg, s):
    """With amax = 448 s the block scale is s; x = m * s (exact in bf16 for every e4m3 midpoint m)
    makes x / s exactly a midpoint, a tie that x * RN(1/s) misses by an ulp: the kernel must still
    round the exact quotient (to even), as the oracle does.  Neighbouring bf16 values included."""
    d = oracle.e4m3_decode_table()
    mids = (d[0:0x7E] + d[1:0x7F]) / 2
    vals = np.concatenate([mids * s, np.nextafter(mids * s, np.inf), -mids * s]).astype(np.float32)
    vals = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()  # the neighbours become bf16 values
    per_row = 127
    nrows = (len(vals) + per_row - 1) // per_row
    x = np.zeros((nrows, 128), dtype=np.float32)
    x[:, 0] = 448.0 * s  # the block maximum fixes the scale at exactly s
    flat = np.zeros(nrows * per_row, dtype=np.float32)
    flat[:len(vals)] = vals
    x[:, 1:] = flat.reshape(nrows, per_row)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(x))  # every value is exact in bf16
    q, sfa = fg.cast_fp8_rows(xb.cuda())
    torch.cuda.synchronize()
    q_ref, sfa_ref = oracle.quantize_rows(as_bits(xb))
    assert np.all(sfa_ref[0, :nrows] == np.float32(s))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sfa.cpu().numpy()[:, :nrows], sfa_ref[:, :nrows])


@pytest.mark.parametrize("shape", [(7, 272), (33, 1040), (2, 129, 384)])
def test_cast_e5m2_bit_exact(fg, shape):
    x = bf16_inputs(shape, 3 * sum(shape))
    q, s = fg.cast_fp8_rows(x.cuda(), fmt="e5m2")
    qb, sb = fg.cast_fp8_blocks(x.cuda(), fmt="e5m2")
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_rows(as_bits(x), fmt="e5m2")
    qb_ref, sb_ref = oracle.quantize_blocks(as_bits(x), fmt="e5m2")
    M = shape[-2]
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy()[..., :M].view(np.uint32), s_ref[..., :M].view(np.uint32))
    assert np.array_equal(qb.cpu().numpy(), qb_ref)
    assert np.array_equal(sb.cpu().numpy().view(np.uint32), sb_ref.view(np.uint32))


def test_cast_e5m2_quotients_on_midpoints(fg):
    d = oracle.e5m2_decode_table()
    mids = (d[0:0x7B] + d[1:0x7C]) / 2
    s = 1.5  # amax = 57344 * 1.5 makes the scale exactly 1.5; m * 1.5 is exact in bf16
    vals = np.concatenate([mids * s, -mids * s]).astype(np.float32)
    per_row = 127
    nrows = (len(vals) + per_row - 1) // per_row
    x = np.zeros((nrows, 128), dtype=np.float32)
    x[:, 0] = 57344.0 * s
    flat = np.zeros(nrows * per_row, dtype=np.float32)
    flat[:len(vals)] = vals
    x[:, 1:] = flat.reshape(nrows, per_row)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(x))
    q, sfa = fg.cast_fp8_rows(xb.cuda(), fmt="e5m2")
    torch.cuda.synchronize()
    q_ref, sfa_ref = oracle.quantize_rows(as_bits(xb), fmt="e5m2")
    assert np.all(sfa_ref[0, :nrows] == np.float32(s))
    assert np.array_equal(q.cpu().numpy(), q_ref)
