"""The tile table (fg_tile_plan): the kernel and tile width each large-M call takes.  N <= 128
and N <= 192 take the one-CTA kernel at that width; the contiguous and masked layouts the one-CTA
256-wide kernel; dense calls the 256 x 256 CTA pair unless its last wave of tiles holds at most a
quarter of the SM pairs (then the one-CTA kernel, whose stream-K tail splits that wave).  The
overrides (fg_set_dense_path, fg_set_tile_n) and the small-M answer (2000) are checked too.
"""
from __future__ import annotations

import pytest
import torch

from synth import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_dense_path(0)
    lib.set_tile_n(0)


def expected_dense(M, N, sms):
    if N <= 128:
        return 1128
    if N <= 192:
        return 1192
    pairs = max(sms // 2, 1)
    rem = (-(-M // 256) * -(-N // 256)) % pairs
    return 1256 if rem != 0 and rem * 4 <= pairs else 3256


def test_table_on_the_benchmark_shapes(fg):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for w in workloads.prefill():
        assert fg.tile_plan("dense", w["M"], w["N"], w["K"], 1) == expected_dense(w["M"], w["N"], sms), w["name"]
    for w in workloads.contiguous():
        assert fg.tile_plan("contiguous", w["M_per_group"] * w["G"], w["N"], w["K"], w["G"]) == 1256, w["name"]
    for w in workloads.masked():
        assert fg.tile_plan("masked", w["Mmax"], w["N"], w["K"], w["G"]) == 1256, w["name"]
    for w in workloads.decode_sweep():
        assert fg.tile_plan("dense", w["M"], w["N"], w["K"], 1) == 2000, w["name"]


@pytest.mark.parametrize("M,N", [(300, 128), (4096, 136), (513, 192), (1024, 200), (4096, 7168), (4096, 2112)])
def test_table_rule(fg, M, N):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fg.tile_plan("dense", M, N, 1024, 1) == expected_dense(M, N, sms)
    assert fg.tile_plan("contiguous", M, N, 1024, 2) == (1128 if N <= 128 else 1192 if N <= 192 else 1256)


def test_table_overrides(fg):
    old_path, old_n = fg.set_dense_path(1), fg.set_tile_n(0)
    try:
        assert fg.tile_plan("dense", 4096, 4096, 7168, 1) == 1256  # the one-CTA kernel forced
        assert fg.tile_plan("dense", 64, 4096, 7168, 1) == 1256   # also below M = 129
        fg.set_dense_path(3)
        assert fg.tile_plan("dense", 4096, 7168, 16384, 1) == 3256  # the pair forced
        assert fg.tile_plan("contiguous", 4096, 4096, 7168, 4) == 1256  # never the pair for contiguous
        fg.set_tile_n(128)
        assert fg.tile_plan("dense", 4096, 4096, 7168, 1) == 3192  # the pair has 192 and 256 only
        fg.set_dense_path(1)
        assert fg.tile_plan("masked", 256, 4096, 7168, 4) == 1128
        fg.set_dense_path(2)
        assert fg.tile_plan("dense", 4096, 4096, 7168, 1) == 2000
    finally:
        fg.set_dense_path(old_path)
        fg.set_tile_n(old_n)
