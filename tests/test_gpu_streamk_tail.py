"""GPU parity of the tiled kernel's stream-K tail (the last partial wave of tiles split in K over
all CTAs, split tiles summed by the last CTA to finish) against the CPU oracle.

The threshold is forced to 0 (split whenever it is not longer), so small odd shapes take the tail
with many pieces per tile, single-K-block pieces, tiles shared by more CTAs than K blocks, dead
tiles of the contiguous layout and a masked walk whose tail is decided on the device; -1 turns
the tail off.  The default threshold is exercised by the full-size workloads of
test_gpu_parity.py.  Tolerance as there (tests/gpu_helpers.py).
"""
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
    yield lib
    lib.set_dense_path(0)


class streamk:
    """Context manager: tiled-kernel stream-K threshold (and the tiled path for dense calls)."""

    def __init__(self, fg, overhead):
        self.fg, self.overhead = fg, overhead

    def __enter__(self):
        self.old = self.fg.set_tiled_streamk(self.overhead)
        self.old_path = self.fg.set_dense_path(1)

    def __exit__(self, *exc):
        self.fg.set_tiled_streamk(self.old)
        self.fg.set_dense_path(self.old_path)


def canary_like(shape):
    return torch.full(shape, -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def dense(fg, case, overhead):
    with streamk(fg, overhead):
        A, sfa, B, sfb = dense_dev(case)
        C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
        torch.cuda.synchronize()
    return bits_of(C)


# (M, N, K): tiles of 128 x 192, K blocks of 128
SHAPES = [
    (129, 520, 256),     # 6 tiles, 2 K blocks: one-block pieces, 2 per tile
    (300, 392, 1152),    # 9 tiles, 9 K blocks: 9 pieces per tile
    (200, 136, 128),     # 2 tiles, 1 K block: every piece is a whole tile
    (513, 2048, 3072),   # 55 tiles over 148 CTAs: pieces of 8-9 K blocks
    (1000, 4104, 1024),  # 176 tiles: one whole wave, then 28 tiles split
    (4096, 2112, 512),   # 352 tiles: two whole waves, 56 tiles split over 148 CTAs
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_dense_tail_forced_and_off(fg, M, N, K):
    case = synth.dense_case(700 + M, M, N, K, row_scaled=True)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    got = dense(fg, case, 0)
    close(got, ref, f"tail forced {M}x{N}x{K}")
    close(dense(fg, case, -1), ref, f"tail off {M}x{N}x{K}")
    # bit-reproducible: the pieces are summed in CTA order whatever CTA finishes last
    for _ in range(2):
        np.testing.assert_array_equal(dense(fg, case, 0), got)


def test_dense_tail_default_threshold_full_wave(fg):
    """2048 x 2112 x 7168: 176 tiles, the 28 past the first wave are split at the default threshold."""
    case = synth.dense_case(777, 2048, 2112, 7168)
    rows = np.unique(np.concatenate([np.arange(0, 2048, 61), [2047, 1920, 1919]])).astype(np.int32)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], rows=rows)
    got = dense(fg, case, 8)
    close(got[rows], ref, "default threshold")
    np.testing.assert_array_equal(dense(fg, case, 8), got)


def test_contiguous_tail_with_padding(fg):
    case = synth.contiguous_case(741, [100, 0, 300, 37, 128, 1], N=264, K=1152)
    A, sfa = to_dev(case["A"]), to_dev(case["sfa"])
    B, sfb = to_dev(case["B"]), to_dev(case["sfb"])
    mi = to_dev(case["m_indices"])
    canary = np.full((case["M"], case["N"]), 0xFFFF, dtype=np.uint16)
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"], C=canary)
    live = case["m_indices"] >= 0
    for overhead in (0, -1):
        C = canary_like((case["M"], case["N"]))
        with streamk(fg, overhead):
            fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(A, sfa, B, sfb, mi, C=C)
            torch.cuda.synchronize()
        got = bits_of(C)
        close(got[live], ref[live], f"contiguous tail overhead={overhead}")
        assert np.all(got[~live] == 0xFFFF), "padding rows were written"


def test_masked_tail_decided_on_device(fg):
    """The live tile count comes from masked_m on the device; one CUDA graph, replayed with counts
    that give no tail, a tail, and no tiles at all."""
    G, Mmax, N, K = 4, 384, 1000, 1536
    case = synth.masked_case(751, G, Mmax, N, K, masked_m=[384, 0, 129, 7])
    A, sfa, B, sfb = to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]), to_dev(case["sfb"])
    mm = to_dev(case["masked_m"])
    C = canary_like((G, Mmax, N))
    with streamk(fg, 0):
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)  # warm-up outside capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)
        for counts in ([384, 0, 129, 7], [384, 384, 384, 384], [1, 0, 0, 300], [0, 0, 0, 0]):
            counts = np.array(counts, dtype=np.int32)
            mm.copy_(torch.from_numpy(counts).cuda())
            C.view(torch.int16).fill_(-1)
            graph.replay()
            torch.cuda.synchronize()
            got = bits_of(C)
            canary = np.full((G, Mmax, N), 0xFFFF, dtype=np.uint16)
            ref = oracle.grouped_masked(case["A"], case["sfa"], case["B"], case["sfb"], counts, C=canary)
            for g in range(G):
                v = int(counts[g])
                if v:
                    close(got[g, :v], ref[g, :v], f"masked tail {counts.tolist()} g={g}")
                assert np.all(got[g, v:] == 0xFFFF), f"rows past masked_m[{g}] were written"
        del graph
    assert fg.device_status() == 0
