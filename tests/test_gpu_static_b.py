"""FG_FLAG_STATIC_B on the GPU: the small-M kernel loads the weight half of its first ring stages
before waiting for the preceding kernel.  The arithmetic is unchanged, so outputs must be
bit-identical to the stream-ordered call on every schedule, alone and in a chain of back-to-back
launches replayed from a CUDA graph (where each launch's early weight loads overlap the previous
launch); and they must match the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import bits_of, close, dense_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_swap_schedule(0)


@pytest.mark.parametrize("schedule", [0, -1, 1, 2])
@pytest.mark.parametrize("M,N,K", [(64, 2112, 7168), (128, 7168, 2048), (7, 264, 384), (33, 24576, 1536)])
def test_static_b_is_bit_identical(fg, schedule, M, N, K):
    case = synth.dense_case(600 + M, M, N, K, row_scaled=True)
    A, sfa, B, sfb = dense_dev(case)
    old = fg.set_swap_schedule(schedule)
    try:
        plain = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
        early = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, static_b=True))
    finally:
        fg.set_swap_schedule(old)
    np.testing.assert_array_equal(early, plain)
    if schedule == 0:
        close(early, oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"]), f"static_b {M}x{N}x{K}")


def test_static_b_chain_under_cuda_graph(fg):
    """The twelve decode-sweep GEMMs back to back in one graph, each output then fed to nothing:
    early weight loads of launch i+1 overlap launch i; replayed twice, every output exact."""
    cases = [synth.dense_case(w["seed"], w["M"], w["N"], w["K"], row_scaled=True) for w in workloads.decode_sweep()]
    devs = [dense_dev(c) for c in cases]
    plain = [bits_of(fg.gemm_fp8_fp8_bf16_nt(*d)) for d in devs]
    outs = [torch.empty((c["M"], c["N"]), dtype=torch.bfloat16, device="cuda") for c in cases]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for d, o in zip(devs, outs):
            fg.gemm_fp8_fp8_bf16_nt(*d, C=o, static_b=True)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for d, o in zip(devs, outs):
            fg.gemm_fp8_fp8_bf16_nt(*d, C=o, stream=s, static_b=True)
    for _ in range(2):
        for o in outs:
            o.view(torch.int16).fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        for o, p in zip(outs, plain):
            np.testing.assert_array_equal(bits_of(o), p)
    del g
    close(plain[0], oracle.gemm_nt(cases[0]["A"], cases[0]["sfa"], cases[0]["B"], cases[0]["sfb"]), "chain[0]")
