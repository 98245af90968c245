"""Non-finite input codes on the GPU, against the oracle's IEEE reading (the pages say nothing
about NaN or infinite inputs; the oracle propagates them by IEEE rules, pinned on the CPU by
tests/test_oracle_specials.py): an e4m3 NaN code (0x7F / 0xFF) or an e5m2 NaN makes every output
it enters NaN, an e5m2 infinity gives an infinity with the sign of the product, infinity times
zero and opposite infinities in one sum give NaN.  Checked on every kernel and layout: the NaN
and infinity positions must match the oracle's exactly, the finite rest within the tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close_nonfinite, dense_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_dense_path(0)
    lib.set_swap_schedule(0)


def plant(A2, B2, fmt, seed):
    """Write special codes into 2-D views of A and B (in place)."""
    rng = np.random.default_rng(seed)
    M, K = A2.shape
    N = B2.shape[0]
    if fmt == "e4m3":
        A2[rng.integers(M), rng.integers(K)] = 0x7F                   # NaN row
        B2[rng.integers(N), rng.integers(K)] = 0xFF                   # NaN column
    else:
        m1, m2 = rng.choice(M, 2, replace=False) if M > 1 else (0, 0)
        A2[m1, rng.integers(K)] = 0x7C                                # +inf: row of infinities / NaN where x0
        A2[m2, 3] = 0xFC                                              # -inf in the first K block ...
        A2[m2, K - 5] = 0x7C                                          # ... and +inf in the last: NaN if KB > 1
        B2[rng.integers(N), rng.integers(K)] = 0x7E                   # NaN column
        n0 = rng.integers(N)
        k0 = rng.integers(K)
        B2[n0, k0] = 0xFC                                             # -inf column ...
        A2[:, k0] = np.where(np.arange(M) % 3 == 0, 0x00, A2[:, k0])  # ... meeting zeros (NaN) in some rows


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("M,N,K,path,schedule", [
    (200, 520, 1152, 1, 0),    # one-CTA tiled
    (300, 392, 640, 3, 0),     # CTA pair
    (64, 2112, 1536, 2, -1),   # swap-AB stream-K
    (64, 2112, 1536, 2, 4),    # swap-AB cluster split
    (33, 520, 896, 2, 1),      # swap-AB whole tiles
])
def test_dense_special_codes(fg, fmt, M, N, K, path, schedule):
    case = synth.dense_case(70 + M, M, N, K, fmt_a=fmt, fmt_b=fmt)
    plant(case["A"], case["B"], fmt, M + N)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], fmt_a=fmt, fmt_b=fmt)
    A, sfa, B, sfb = dense_dev(case)
    old, old_s = fg.set_dense_path(path), fg.set_swap_schedule(schedule)
    try:
        C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, fmt_a=fmt, fmt_b=fmt)
        torch.cuda.synchronize()
    finally:
        fg.set_dense_path(old)
        fg.set_swap_schedule(old_s)
    st = close_nonfinite(bits_of(C), ref, f"{fmt} {M}x{N}x{K} path {path} schedule {schedule}")
    assert st["nan"] > 0


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_grouped_special_codes(fg, fmt):
    cc = synth.contiguous_case(81, [100, 0, 300], N=264, K=640, fmt_a=fmt, fmt_b=fmt)
    plant(cc["A"], cc["B"][2], fmt, 1)
    C = torch.full((cc["M"], cc["N"]), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(to_dev(cc["A"]), to_dev(cc["sfa"]), to_dev(cc["B"]),
                                                  to_dev(cc["sfb"]), to_dev(cc["m_indices"]), C=C,
                                                  fmt_a=fmt, fmt_b=fmt)
    torch.cuda.synchronize()
    live = cc["m_indices"] >= 0
    ref = oracle.grouped_contiguous(cc["A"], cc["sfa"], cc["B"], cc["sfb"], cc["m_indices"], fmt_a=fmt, fmt_b=fmt)
    close_nonfinite(bits_of(C)[live], ref[live], f"contiguous {fmt}")

    mc = synth.masked_case(82, 2, 256, 264, 640, masked_m=[77, 256], fmt_a=fmt, fmt_b=fmt)
    plant(mc["A"][1], mc["B"][1], fmt, 2)
    plant(mc["A"][0, :77], mc["B"][0], fmt, 3)
    C = torch.full((2, 256, 264), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(to_dev(mc["A"]), to_dev(mc["sfa"]), to_dev(mc["B"]), to_dev(mc["sfb"]),
                                              to_dev(mc["masked_m"]), C=C, fmt_a=fmt, fmt_b=fmt)
    torch.cuda.synchronize()
    ref = oracle.grouped_masked(mc["A"], mc["sfa"], mc["B"], mc["sfb"], mc["masked_m"], fmt_a=fmt, fmt_b=fmt)
    got = bits_of(C)
    close_nonfinite(got[0, :77], ref[0, :77], f"masked {fmt} g=0")
    close_nonfinite(got[1], ref[1], f"masked {fmt} g=1")
    assert (got[0, 77:] == 0xFFFF).all()
