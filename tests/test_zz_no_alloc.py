"""The allocation-free entry point, fp8_gemm_nt_noalloc.

It exists for callers that cannot allocate device memory themselves (a framework's
memory pool owns the device, a static memory plan, or a decode step that must not
touch the allocator).  It keeps its split-K scratch in a static device array, so
these tests call it through the C ABI with plain device pointers and check it
against the regular entry point, fp8_gemm_nt, with the tolerance every parity test
uses -- twice in a row, since both calls share the one array.  This file is named so
that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import synth
from tests.gpu_helpers import bits_of, close, dense_dev

pytestmark = pytest.mark.gpu

SHAPES = [(64, 2112, 7168), (128, 4096, 2048), (7, 264, 384), (33, 7168, 512)]


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_noalloc_matches_default_entry_point_twice(M, N, K):
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    fg.init(0)
    case = synth.dense_case(900 + M, M, N, K, row_scaled=True)
    A, sfa, B, sfb = dense_dev(case)
    ref = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
    for call in range(2):
        C = torch.full((M, N), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        rc = fg.lib.fp8_gemm_nt_noalloc(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(),
                                        M, N, K, _stream())
        assert rc == 0, fg.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        close(bits_of(C), ref, f"noalloc call {call} {M}x{N}x{K}")
    assert fg.lib.fg_noalloc_status(_stream()) == 0


def test_noalloc_rejects_sizes_beyond_its_limits():
    import moe_grouped_gemm_08_b200 as fg
    p = 0x10000  # never dereferenced: the size checks come first
    assert fg.lib.fp8_gemm_nt_noalloc(p, p, p, p, p, 129, 256, 128, None) == 3   # M > 128
    assert fg.lib.fp8_gemm_nt_noalloc(p, p, p, p, p, 64, 16384 * 128 + 8, 128, None) == 3  # too many n-tiles
