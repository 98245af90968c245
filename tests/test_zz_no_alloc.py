"""The allocation-free entry point, fp8_gemm_nt_noalloc.

It exists for callers that cannot allocate device memory themselves (a framework's
memory pool owns the device, a static memory plan, or a decode step that must not
touch the allocator).  It keeps its split-K scratch in a static device array, so
these tests call it through the C ABI with plain device pointers and check it, with
the tolerance every parity test uses, against the CPU oracle and against the regular
entry point, fp8_gemm_nt -- twice in a row, since both calls share the one array.
The timeout path of the variant is exercised with the stall hook, without a fault.
This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes
import time

import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close, dense_dev

pytestmark = pytest.mark.gpu

SHAPES = [(64, 2112, 7168), (128, 4096, 2048), (7, 264, 384), (33, 7168, 512)]
FG_ERR_TIMEOUT = 6


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(fg, A, sfa, B, sfb, M, N, K):
    C = torch.full((M, N), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    rc = fg.lib.fp8_gemm_nt_noalloc(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(),
                                    M, N, K, _stream())
    assert rc == 0, fg.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    return bits_of(C)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_noalloc_matches_oracle_and_default_entry_point_twice(M, N, K):
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    fg.init(0)
    case = synth.dense_case(900 + M, M, N, K, row_scaled=True)
    A, sfa, B, sfb = dense_dev(case)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    regular = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
    close(regular, ref, f"fp8_gemm_nt {M}x{N}x{K}")
    for call in range(2):
        got = _noalloc(fg, A, sfa, B, sfb, M, N, K)
        close(got, ref, f"noalloc call {call} {M}x{N}x{K} vs oracle")
        close(got, regular, f"noalloc call {call} {M}x{N}x{K} vs fp8_gemm_nt")
    assert fg.lib.fg_noalloc_status(_stream()) == 0


def test_noalloc_timeout_is_reported_and_next_call_is_clean():
    """The stall hook makes the variant's bounded wait run out (about two seconds, no trap); its
    own status word reports FG_ERR_TIMEOUT once, and the next call is correct with a clean word."""
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    M, N, K = 64, 7168, 16384  # 48 K blocks per CTA: more than the ring holds
    case = synth.dense_case(61, M, N, K, row_scaled=True)
    A, sfa, B, sfb = dense_dev(case)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    _noalloc(fg, A, sfa, B, sfb, M, N, K)  # first call on the device: looks up the array's address
    assert fg.lib.fg_noalloc_status(_stream()) == 0
    old = fg.lib.fg_debug_set_stall(1)
    try:
        t0 = time.time()
        _noalloc(fg, A, sfa, B, sfb, M, N, K)
        status = fg.lib.fg_noalloc_status(_stream())
        elapsed = time.time() - t0
    finally:
        fg.lib.fg_debug_set_stall(old)
    assert status == FG_ERR_TIMEOUT, fg.STATUS_NAMES.get(status, status)
    assert 1.0 < elapsed < 20.0, elapsed
    assert fg.lib.fg_noalloc_status(_stream()) == 0  # cleared by the read
    for call in range(2):
        close(_noalloc(fg, A, sfa, B, sfb, M, N, K), ref, f"noalloc after the timeout, call {call}")
    assert fg.lib.fg_noalloc_status(_stream()) == 0


def test_noalloc_rejects_sizes_beyond_its_limits():
    import moe_grouped_gemm_08_b200 as fg
    p = 0x10000  # never dereferenced: the size checks come first
    assert fg.lib.fp8_gemm_nt_noalloc(p, p, p, p, p, 129, 256, 128, None) == 3   # M > 128
    assert fg.lib.fp8_gemm_nt_noalloc(p, p, p, p, p, 64, 16384 * 128 + 8, 128, None) == 3  # too many n-tiles
