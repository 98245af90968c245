"""CPU checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments on the host before touching the GPU."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

import moe_grouped_gemm_08_b200 as fg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8gemm.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("fp8_gemm_nt", "fp8_gemm_grouped_contiguous", "fp8_gemm_grouped_masked", "fg_init",
                     "fg_m_alignment", "fg_sfa_ld", "fg_get_device_status", "fg_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(str(fg.LIB_PATH))
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in fp8gemm.h but not exported"


def test_queries():
    assert fg.get_m_alignment_for_contiguous_layout() == 128
    assert [fg.sfa_ld(m) for m in (0, 1, 4, 5, 128, 1025)] == [0, 4, 4, 8, 128, 1028]
    assert fg.STATUS_NAMES[6] == "FG_ERR_TIMEOUT"
    assert fg.lib.fg_status_string(99) == b"FG_ERR_UNKNOWN"


def test_dense_path_switch():
    old = fg.set_dense_path(1)
    assert fg.set_dense_path(2) == 1
    assert fg.set_dense_path(3) == 2
    assert fg.set_dense_path(7) == 3  # ignored
    fg.set_dense_path(old)


def test_schedule_switches():
    old = fg.set_swap_schedule(4)
    assert old == 0  # automatic by default
    assert fg.set_swap_schedule(-1) == 4
    assert fg.set_swap_schedule(3) == -1  # not a cluster size: ignored
    assert fg.set_swap_schedule(8) == -1
    assert fg.set_swap_schedule(1) == 8
    fg.set_swap_schedule(old)
    old = fg.set_tiled_streamk(0)
    assert old == 18  # default cost charged for publishing partial tiles, in K blocks
    assert fg.set_tiled_streamk(-5) == 0
    assert fg.set_tiled_streamk(old) == -1  # any negative value is stored as -1 (never split)
    old = fg.set_tile_order(1)
    assert old == 0  # automatic by default (by the bytes of one group's B)
    assert fg.set_tile_order(2) == 1
    assert fg.set_tile_order(3) == 2  # not a walk: ignored
    assert fg.set_tile_order(-1) == 2
    assert fg.set_tile_order(old) == 2


def test_swap_plan_without_device_state():
    # no fg_init on a machine without a GPU: the query answers -1 and launches nothing
    if not torch.cuda.is_available():
        assert fg.swap_plan(64, 2112, 7168) == -1
    assert fg.swap_plan(0, 2112, 7168) == -1
    assert fg.swap_plan(129, 2112, 7168) == -1


NULL = None
P16 = 0x10000  # a fake 16-byte-aligned address: these calls must fail before any dereference


@pytest.mark.parametrize("args,expect", [
    ((NULL, P16, P16, P16, P16, 64, 128, 128, NULL), 1),     # null A
    ((P16, P16, P16, P16, P16, 64, 128, 0, NULL), 1),        # K = 0
    ((P16, P16, P16, P16, P16, -1, 128, 128, NULL), 1),      # negative M
    ((P16, P16, P16, P16, P16, 64, 128, 120, NULL), 2),      # K % 16
    ((P16, P16, P16, P16, P16, 64, 100, 128, NULL), 2),      # N % 8
    ((P16 + 8, P16, P16, P16, P16, 64, 128, 128, NULL), 2),  # A misaligned
    ((P16, P16 + 2, P16, P16, P16, 64, 128, 128, NULL), 2),  # sfa misaligned
    ((P16, P16, P16, P16, P16, 0, 128, 128, NULL), 0),       # M = 0: no-op
    ((NULL, NULL, NULL, NULL, NULL, 0, 0, 0, NULL), 0),      # empty: no-op
])
def test_dense_argument_errors(args, expect):
    assert fg.lib.fp8_gemm_nt(*args) == expect


def test_grouped_argument_errors():
    L = fg.lib
    assert L.fp8_gemm_grouped_contiguous(P16, P16, P16, P16, P16, NULL, 256, 2, 128, 128, NULL) == 1
    assert L.fp8_gemm_grouped_contiguous(P16, P16, P16, P16, P16, P16, 256, 0, 128, 128, NULL) == 1
    assert L.fp8_gemm_grouped_contiguous(P16, P16, P16, P16, P16, P16 + 2, 256, 2, 128, 128, NULL) == 2
    assert L.fp8_gemm_grouped_contiguous(P16, P16, P16, P16, P16, P16, 0, 2, 128, 128, NULL) == 0
    assert L.fp8_gemm_grouped_masked(P16, P16, P16, P16, P16, NULL, 2, 64, 128, 128, NULL) == 1
    assert L.fp8_gemm_grouped_masked(P16, P16, P16, P16, P16, P16, 2000, 64, 128, 128, NULL) == 3
    assert L.fp8_gemm_grouped_masked(P16, P16, P16, P16, P16, P16, 2, 64, 128, 136, NULL) == 2
    assert L.fp8_gemm_grouped_masked(P16, P16, P16, P16, P16, P16, 0, 64, 128, 128, NULL) == 0


def test_cast_argument_errors():
    cast_rows, cast_blocks = fg.lib.fp8_cast_rows, fg.lib.fp8_cast_blocks
    for f in (cast_rows, cast_blocks):
        assert f(NULL, P16, P16, 1, 4, 128, NULL) == 1           # null input
        assert f(P16, P16, P16, 1, 4, -128, NULL) == 1           # negative K
        assert f(P16, P16, P16, 1, 4, 120, NULL) == 2            # K % 16
        assert f(P16 + 8, P16, P16, 1, 4, 128, NULL) == 2        # X not 16-byte aligned
        assert f(P16, P16 + 4, P16, 1, 4, 128, NULL) == 2        # Q not 16-byte aligned
        assert f(P16, P16, P16, 0, 4, 128, NULL) == 0            # G = 0: no-op, nothing launched
        assert f(P16, P16, P16, 1, 0, 128, NULL) == 0            # no rows: no-op
    assert cast_blocks(P16, P16, P16, 70000, 4, 128, NULL) == 3  # more groups than a grid axis holds


def test_debug_build_exports_the_same_symbols():
    lib = fg.debug_library()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from the debug build"
    assert fg.STATUS_NAMES[7] == "FG_ERR_DEVICE_CHECK"
    assert lib.fg_status_string(7) == b"FG_ERR_DEVICE_CHECK"


def test_workspace_entry_points_check_arguments_first():
    L = fg.lib
    if not torch.cuda.is_available():
        assert L.fg_workspace_bytes() == 0  # no fg_init on this device
        # arguments valid, no device state: not initialised, nothing launched
        assert L.fp8_gemm_nt_ws(P16, P16, P16, P16, P16, 64, 128, 128, 0, 0, 1, P16, 1 << 30, NULL) == 4
    assert L.fp8_gemm_nt_ws(P16, P16, P16, P16, P16, 64, 128, 120, 0, 0, 0, P16, 1 << 30, NULL) == 2   # K % 16
    assert L.fp8_gemm_nt_ws(P16, P16, P16, P16, P16, 64, 128, 128, 2, 0, 0, P16, 1 << 30, NULL) == 1   # format
    assert L.fp8_gemm_nt_ws(P16, P16, P16, P16, P16, 64, 128, 128, 0, 0, 6, P16, 1 << 30, NULL) == 1   # flag
    assert L.fp8_gemm_grouped_contiguous_ws(P16, P16, P16, P16, P16, NULL, 256, 2, 128, 128, 0, 0, 0, P16, 1 << 30,
                                            NULL) == 1
    assert L.fp8_gemm_grouped_masked_ws(P16, P16, P16, P16, P16, P16, 2000, 64, 128, 128, 0, 0, 0, P16, 1 << 30,
                                        NULL) == 3
    assert L.fp8_gemm_nt_ws(P16, P16, P16, P16, P16, 0, 128, 128, 0, 0, 0, NULL, 0, NULL) == 0  # M = 0: no-op


def test_runtime_specialisation_compiles_without_a_gpu():
    """The runtime-specialisation path compiles the tiled kernel for sm_100a from the sources
    embedded in the library (NVRTC; no GPU needed), for each tile width."""
    for bn in (128, 192, 256):
        assert fg.jit_compile_check(bn, 56, 4096) > 100_000
    assert fg.lib.fg_jit_compile_check(100, 56, 4096, ctypes.byref(ctypes.c_size_t())) == 1  # bad width
    old = fg.set_jit(True)
    assert fg.set_jit(bool(old)) == 1
