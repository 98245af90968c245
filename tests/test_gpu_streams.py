"""GEMMs on two streams at once, each stream with its own caller-owned workspace (the _ws entry
points): split-K schedules on both (the small-M kernel's stream-K fix-up and the tiled kernel's
stream-K tail), launched alternately so that the kernels overlap; every output must match the
oracle and be bit-identical across repetitions."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bits_of, close, dense_dev, to_dev

pytestmark = pytest.mark.gpu


def test_two_streams_with_their_own_workspaces():
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    fg.init(0)
    ca = synth.dense_case(501, 64, 7168, 16384, row_scaled=True)   # swap-AB kernel, stream-K forced
    cb = synth.dense_case(502, 300, 4096, 7168)                     # tiled kernel, stream-K tail forced
    cc = synth.contiguous_case(503, [200, 300], N=2112, K=2048)      # contiguous, tail forced
    ra = oracle.gemm_nt(ca["A"], ca["sfa"], ca["B"], ca["sfb"])
    rb = oracle.gemm_nt(cb["A"], cb["sfa"], cb["B"], cb["sfb"])
    rc = oracle.grouped_contiguous(cc["A"], cc["sfa"], cc["B"], cc["sfb"], cc["m_indices"])
    da, db = dense_dev(ca), dense_dev(cb)
    dc = [to_dev(cc[k]) for k in ("A", "sfa", "B", "sfb", "m_indices")]
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    w1, w2 = fg.new_workspace(), fg.new_workspace()
    assert w1.numel() == fg.workspace_bytes() > 0
    reps = 12
    outs_a = [torch.empty((64, 7168), dtype=torch.bfloat16, device="cuda") for _ in range(reps)]
    outs_b = [torch.empty((300, 4096), dtype=torch.bfloat16, device="cuda") for _ in range(reps)]
    outs_c = [torch.empty((cc["M"], cc["N"]), dtype=torch.bfloat16, device="cuda") for _ in range(reps)]
    old = (fg.set_swap_schedule(-1), fg.set_tiled_streamk(0))
    try:
        assert fg.swap_plan(64, 7168, 16384) == 0  # stream-K
        torch.cuda.synchronize()
        for i in range(reps):
            with torch.cuda.stream(s1):
                fg.gemm_fp8_fp8_bf16_nt(*da, C=outs_a[i], workspace=w1)
                if i % 2:
                    fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(*dc, C=outs_c[i], workspace=w1)
            with torch.cuda.stream(s2):
                fg.gemm_fp8_fp8_bf16_nt(*db, C=outs_b[i], workspace=w2)
                if not i % 2:
                    fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(*dc, C=outs_c[i], workspace=w2)
        torch.cuda.synchronize()
    finally:
        fg.set_swap_schedule(old[0])
        fg.set_tiled_streamk(old[1])
    assert fg.device_status() == 0
    live = cc["m_indices"] >= 0
    first = [bits_of(outs_a[0]), bits_of(outs_b[0]), bits_of(outs_c[0])]
    close(first[0], ra, "stream 1 swap-AB")
    close(first[1], rb, "stream 2 tiled")
    close(first[2][live], rc[live], "contiguous")
    for i in range(1, reps):
        np.testing.assert_array_equal(bits_of(outs_a[i]), first[0])
        np.testing.assert_array_equal(bits_of(outs_b[i]), first[1])
        np.testing.assert_array_equal(bits_of(outs_c[i])[live], first[2][live])
    # the caller's workspaces hold zero counters again
    nb = fg.workspace_bytes()
    for w in (w1, w2):
        assert int(w[nb - 65536 * 4:].view(torch.int32).abs().sum()) == 0


def test_workspace_too_small_is_rejected():
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    fg.init(0)
    case = synth.dense_case(504, 64, 256, 256)
    A, sfa, B, sfb = dense_dev(case)
    small = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    before = fg.launch_count()
    with pytest.raises(fg.FP8GemmError):
        fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, workspace=small)
    assert fg.launch_count() == before
