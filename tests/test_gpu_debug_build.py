"""The debug build (libfp8gemm_debug.so, -DFG_DEBUG) on the GPU: its device-side index checks
report FG_ERR_DEVICE_CHECK through the status word and never trap; on valid inputs they stay
silent on every kernel and schedule; the release build treats the same bad expert index as
padding without a report."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close, to_dev

pytestmark = pytest.mark.gpu

FG_ERR_DEVICE_CHECK = 7


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _canary(shape):
    return torch.full(shape, -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def _contig(lib, d, C, G):
    M, K = d["A"].shape
    N = d["B"].shape[1]
    return lib.fp8_gemm_grouped_contiguous(d["A"].data_ptr(), d["sfa"].data_ptr(), d["B"].data_ptr(),
                                           d["sfb"].data_ptr(), C.data_ptr(), d["mi"].data_ptr(), M, G, N, K, _s())


def test_out_of_range_expert_index_is_reported_by_the_debug_build_only():
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    dl = fg.debug_library()
    assert dl.fg_init(0) == 0
    fg.init(0)
    case = synth.contiguous_case(42, [128, 128, 128], N=136, K=256)
    mi = case["m_indices"].copy()
    mi[256:384] = 7  # >= G in a whole block
    mi[130] = 9      # >= G inside a live block of expert 1
    d = dict(A=to_dev(case["A"]), sfa=to_dev(case["sfa"]), B=to_dev(case["B"]), sfb=to_dev(case["sfb"]),
             mi=to_dev(mi))
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], mi)
    ok_rows = np.r_[0:130, 131:256]
    for lib, expect in ((dl, FG_ERR_DEVICE_CHECK), (fg.lib, 0)):
        C = _canary((case["M"], case["N"]))
        assert _contig(lib, d, C, 3) == 0
        assert lib.fg_get_device_status(_s()) == expect
        got = bits_of(C)
        close(got[ok_rows], ref[ok_rows], "valid rows")
        assert (got[130] == 0xFFFF).all() and (got[256:] == 0xFFFF).all(), "bad-index rows were written"
        assert lib.fg_get_device_status(_s()) == 0  # cleared by the read
    d["mi"] = to_dev(case["m_indices"])
    C = _canary((case["M"], case["N"]))
    assert _contig(dl, d, C, 3) == 0
    assert dl.fg_get_device_status(_s()) == 0


@pytest.mark.parametrize("M,N,K,path,schedule,tail", [
    (300, 520, 1152, 1, 0, 0),     # tiled kernel, stream-K tail forced
    (300, 392, 640, 3, 0, 18),     # CTA pair
    (64, 7168, 16384, 2, -1, 18),  # swap-AB stream-K
    (64, 2112, 7168, 2, 4, 18),    # swap-AB cluster split
    (128, 24576, 1536, 2, 0, 18),  # swap-AB whole tiles
])
def test_debug_build_is_silent_and_exact_on_valid_inputs(M, N, K, path, schedule, tail):
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    dl = fg.debug_library()
    assert dl.fg_init(0) == 0
    case = synth.dense_case(300 + M, M, N, K, row_scaled=M <= 128)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    A, sfa, B, sfb = (to_dev(case[k]) for k in ("A", "sfa", "B", "sfb"))
    old = (dl.fg_set_dense_path(path), dl.fg_set_swap_schedule(schedule), dl.fg_set_tiled_streamk(tail))
    try:
        C = _canary((M, N))
        assert dl.fp8_gemm_nt(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(), M, N, K,
                              _s()) == 0
        assert dl.fg_get_device_status(_s()) == 0
    finally:
        dl.fg_set_dense_path(old[0])
        dl.fg_set_swap_schedule(old[1])
        dl.fg_set_tiled_streamk(old[2])
    close(bits_of(C), ref, f"debug build {M}x{N}x{K} path {path}")


def test_debug_build_masked_is_silent():
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    dl = fg.debug_library()
    assert dl.fg_init(0) == 0
    mc = synth.masked_case(83, 4, 256, 7168, 2048)
    A, sfa, B, sfb, mm = (to_dev(mc[k]) for k in ("A", "sfa", "B", "sfb", "masked_m"))
    C = _canary((4, 256, 7168))
    assert dl.fp8_gemm_grouped_masked(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(),
                                      mm.data_ptr(), 4, 256, 7168, 2048, _s()) == 0
    assert dl.fg_get_device_status(_s()) == 0
    ref = oracle.grouped_masked(mc["A"], mc["sfa"], mc["B"], mc["sfb"], mc["masked_m"])
    got = bits_of(C)
    for g in range(4):
        v = int(mc["masked_m"][g])
        if v:
            close(got[g, :v], ref[g, :v], f"debug masked g={g}")
        assert (got[g, v:] == 0xFFFF).all()
