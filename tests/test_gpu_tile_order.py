"""GPU parity of the tiled kernels' two tile walks, forced with fg_set_tile_order: m-block groups
(1; A kept in L2) and n-blocks fastest for one m-block at a time (2; B kept in L2), against the CPU
oracle on dense (one-CTA and CTA-pair kernels), contiguous and masked calls that span several
m-blocks and n-blocks with ragged edges.  With the stream-K tail off every tile is computed whole
by one CTA, so the two walks give the same bits.  Tolerance as everywhere (tests/gpu_helpers.py).
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
    lib.set_tile_order(0)
    lib.set_dense_path(0)
    lib.set_tiled_streamk(18)


class settings:
    """Context manager: tile walk, kernel choice and stream-K tail (restored on exit)."""

    def __init__(self, fg, order, path=0, tail=None):
        self.fg, self.order, self.path, self.tail = fg, order, path, tail

    def __enter__(self):
        self.old = (self.fg.set_tile_order(self.order), self.fg.set_dense_path(self.path),
                    self.fg.set_tiled_streamk(self.tail) if self.tail is not None else None)

    def __exit__(self, *exc):
        self.fg.set_tile_order(self.old[0])
        self.fg.set_dense_path(self.old[1])
        if self.old[2] is not None:
            self.fg.set_tiled_streamk(self.old[2])


def canary_like(shape):
    return torch.full(shape, -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)


@pytest.mark.parametrize("path", [1, 3], ids=["tiled", "pair"])
@pytest.mark.parametrize("M,N,K", [(640, 1536, 1024), (1152, 2112, 512), (300, 4104, 768)])
def test_dense_tile_walks(fg, path, M, N, K):
    case = synth.dense_case(1200 + M, M, N, K)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    outs = {}
    for order in (1, 2):
        for tail in (None, -1):
            with settings(fg, order, path, tail):
                A, sfa, B, sfb = dense_dev(case)
                C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
                torch.cuda.synchronize()
            outs[(order, tail)] = bits_of(C)
            close(outs[(order, tail)], ref, f"dense {M}x{N}x{K} path {path} walk {order} tail {tail}")
    np.testing.assert_array_equal(outs[(1, -1)], outs[(2, -1)])


def test_contiguous_tile_walks(fg):
    case = synth.contiguous_case(1301, [300, 0, 520, 128, 77], N=1040, K=512)
    canary = np.full((case["M"], case["N"]), 0xFFFF, dtype=np.uint16)
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"], C=canary)
    live = case["m_indices"] >= 0
    outs = {}
    for order in (1, 2):
        for tail in (None, -1):
            with settings(fg, order, 0, tail):
                C = canary_like((case["M"], case["N"]))
                fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]),
                                                             to_dev(case["sfb"]), to_dev(case["m_indices"]), C=C)
                torch.cuda.synchronize()
            got = bits_of(C)
            close(got[live], ref[live], f"contiguous walk {order} tail {tail}")
            assert np.all(got[~live] == 0xFFFF), "padding rows were written"
            outs[(order, tail)] = got
    np.testing.assert_array_equal(outs[(1, -1)], outs[(2, -1)])


@pytest.mark.parametrize("path", [0, 3], ids=["tiled", "pair"])
def test_masked_tile_walks(fg, path):
    case = synth.masked_case(1401, 3, 384, 776, 640)
    G, Mmax, N = case["G"], case["Mmax"], case["N"]
    canary = np.full((G, Mmax, N), 0xFFFF, dtype=np.uint16)
    ref = oracle.grouped_masked(case["A"], case["sfa"], case["B"], case["sfb"], case["masked_m"], C=canary)
    outs = {}
    for order in (1, 2):
        for tail in (None, -1):
            with settings(fg, order, path, tail):
                C = canary_like((G, Mmax, N))
                fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]),
                                                         to_dev(case["sfb"]), to_dev(case["masked_m"]), C=C)
                torch.cuda.synchronize()
            got = bits_of(C)
            for g in range(G):
                v = min(int(case["masked_m"][g]), Mmax)
                if v:
                    close(got[g, :v], ref[g, :v], f"masked walk {order} tail {tail} g={g}")
                assert np.all(got[g, v:] == 0xFFFF), f"rows past masked_m[{g}]={v} were written"
            outs[(order, tail)] = got
    np.testing.assert_array_equal(outs[(1, -1)], outs[(2, -1)])
