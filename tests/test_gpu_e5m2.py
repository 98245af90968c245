"""GPU parity for E5M2 operands (either or both; the how-to, "Main functions": E4M3 or E5M2
inputs) against the oracle with the same formats, on every kernel: one-CTA tiled, swap-AB
stream-K (M <= 128) and the CTA pair, plus the contiguous and masked layouts.  Tolerance as for
E4M3 (tests/gpu_helpers.close)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close, dense_dev, to_dev

pytestmark = pytest.mark.gpu

PAIRS = [("e5m2", "e5m2"), ("e4m3", "e5m2"), ("e5m2", "e4m3")]


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_dense_path(0)


@pytest.mark.parametrize("fa,fb", PAIRS)
@pytest.mark.parametrize("M,N,K", [(7, 264, 384), (128, 256, 512), (300, 520, 1152)])
def test_dense_e5m2_every_kernel(fg, fa, fb, M, N, K):
    case = synth.dense_case(40 + M, M, N, K, row_scaled=True, fmt_a=fa, fmt_b=fb)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], fmt_a=fa, fmt_b=fb)
    A, sfa, B, sfb = dense_dev(case)
    for path in ([1, 2, 3] if M <= 128 else [1, 3]):
        old = fg.set_dense_path(path)
        try:
            C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, fmt_a=fa, fmt_b=fb)
            torch.cuda.synchronize()
        finally:
            fg.set_dense_path(old)
        close(bits_of(C), ref, f"{fa} x {fb} {M}x{N}x{K} path={path}")


def test_dense_e5m2_decode_shape_from_dtype(fg):
    """float8_e5m2 tensors carry their format through the binding."""
    case = synth.dense_case(71, 64, 2112, 7168, row_scaled=True, fmt_a="e5m2", fmt_b="e5m2")
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], fmt_a="e5m2", fmt_b="e5m2")
    A, sfa, B, sfb = dense_dev(case)
    C = fg.gemm_fp8_fp8_bf16_nt(A.view(torch.float8_e5m2), sfa, B.view(torch.float8_e5m2), sfb)
    torch.cuda.synchronize()
    close(bits_of(C), ref, "e5m2 decode")
    # the same codes read as e4m3 give a different product: the format reaches the MMA
    C4 = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    assert not np.array_equal(bits_of(C4), bits_of(C))


@pytest.mark.parametrize("fa,fb", PAIRS)
def test_contiguous_e5m2(fg, fa, fb):
    case = synth.contiguous_case(43, [100, 0, 300, 37], N=264, K=384, fmt_a=fa, fmt_b=fb)
    C = torch.full((case["M"], case["N"]), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]),
                                                  to_dev(case["sfb"]), to_dev(case["m_indices"]), C=C,
                                                  fmt_a=fa, fmt_b=fb)
    torch.cuda.synchronize()
    got = bits_of(C)
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"],
                                    fmt_a=fa, fmt_b=fb)
    live = case["m_indices"] >= 0
    close(got[live], ref[live], f"contiguous {fa} x {fb}")
    assert np.all(got[~live] == 0xFFFF)


@pytest.mark.parametrize("path", [0, 3], ids=["tiled", "pair"])
@pytest.mark.parametrize("fa,fb", PAIRS)
def test_masked_e5m2(fg, fa, fb, path):
    case = synth.masked_case(53, 3, 200, 264, 384, masked_m=[0, 200, 57], fmt_a=fa, fmt_b=fb)
    C = torch.full((3, 200, 264), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    old = fg.set_dense_path(path)
    try:
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]),
                                                  to_dev(case["sfb"]), to_dev(case["masked_m"]), C=C,
                                                  fmt_a=fa, fmt_b=fb)
        torch.cuda.synchronize()
    finally:
        fg.set_dense_path(old)
    got = bits_of(C)
    ref = oracle.grouped_masked(case["A"], case["sfa"], case["B"], case["sfb"], case["masked_m"],
                                fmt_a=fa, fmt_b=fb)
    close(got[1], ref[1], f"masked {fa} x {fb} g=1")
    close(got[2, :57], ref[2, :57], f"masked {fa} x {fb} g=2")
    assert np.all(got[0] == 0xFFFF) and np.all(got[2, 57:] == 0xFFFF)


def test_invalid_format_is_rejected(fg):
    case = synth.dense_case(3, 8, 136, 256)
    A, sfa, B, sfb = dense_dev(case)
    C = torch.empty((8, 136), dtype=torch.bfloat16, device="cuda")
    rc = fg.lib.fp8_gemm_nt_ex(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(),
                               8, 136, 256, 2, 0, None)
    assert rc == 1  # FG_ERR_INVALID_ARG, nothing launched
