"""Runtime specialisation (fg_set_jit) on the GPU: the one-CTA tiled kernel compiled per shape with
NVRTC, the shape's constants folded in, gives the same bits as the ahead-of-time kernel on the
dense, contiguous and masked layouts and every tile width, matches the oracle, and is compiled once
per shape (cached)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close, dense_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    old = lib.set_dense_path(1)
    yield lib
    lib.set_dense_path(old)
    lib.set_jit(False)
    lib.set_tile_n(0)


def both(fg, fn):
    fg.set_jit(False)
    aot = fn()
    fg.set_jit(True)
    try:
        jit = fn()
    finally:
        fg.set_jit(False)
    return aot, jit


@pytest.mark.parametrize("bn", [128, 192, 256])
@pytest.mark.parametrize("M,N,K", [(300, 520, 1152), (1000, 2112, 7168)])
def test_jit_dense_matches_aot_and_oracle(fg, bn, M, N, K):
    case = synth.dense_case(950 + M, M, N, K)
    A, sfa, B, sfb = dense_dev(case)
    old = fg.set_tile_n(bn)
    try:
        def run():
            C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
            torch.cuda.synchronize()
            return bits_of(C)
        aot, jit = both(fg, run)
        n0 = fg.jit_cache_size()
        fg.set_jit(True)
        again = run()
        fg.set_jit(False)
        assert fg.jit_cache_size() == n0  # compiled once per shape
    finally:
        fg.set_tile_n(old)
    np.testing.assert_array_equal(jit, aot)
    np.testing.assert_array_equal(again, aot)
    rows = np.unique(np.linspace(0, M - 1, 48).astype(np.int32))
    close(jit[rows], oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], rows=rows), f"jit {M}x{N}x{K}")


def test_jit_grouped_layouts_match_aot(fg):
    cc = synth.contiguous_case(961, [200, 0, 300], N=2112, K=2048)
    d = [to_dev(cc[k]) for k in ("A", "sfa", "B", "sfb", "m_indices")]

    def run_c():
        C = torch.full((cc["M"], cc["N"]), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(*d, C=C)
        torch.cuda.synchronize()
        return bits_of(C)
    aot, jit = both(fg, run_c)
    np.testing.assert_array_equal(jit, aot)
    mc = synth.masked_case(962, 4, 256, 4096, 7168)
    dm = [to_dev(mc[k]) for k in ("A", "sfa", "B", "sfb", "masked_m")]

    def run_m():
        C = torch.full((4, 256, 4096), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(*dm, C=C)
        torch.cuda.synchronize()
        return bits_of(C)
    aot, jit = both(fg, run_m)
    np.testing.assert_array_equal(jit, aot)
    assert fg.device_status() == 0
