"""GPU parity of the small-M kernel's cluster split (S CTAs of a thread-block cluster per 128-row
weight tile, each taking 1/S of the K blocks, partials summed through distributed shared memory)
against the CPU oracle, with the schedule forced to each S and compared with the other schedules;
plus the timeout path through the cluster barriers.  Tolerance as in tests/gpu_helpers.py.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import bits_of, close, dense_dev

pytestmark = pytest.mark.gpu

FG_ERR_TIMEOUT = 6


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_swap_schedule(0)
    lib.set_dense_path(0)


def run(fg, case, schedule):
    old = fg.set_swap_schedule(schedule)
    old_path = fg.set_dense_path(2)
    try:
        plan = fg.swap_plan(case["M"], case["N"], case["K"])
        A, sfa, B, sfb = dense_dev(case)
        C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
        torch.cuda.synchronize()
    finally:
        fg.set_swap_schedule(old)
        fg.set_dense_path(old_path)
    return plan, bits_of(C)


# (M, N, K): 128-row weight tiles, K blocks of 128; N % 8 == 0
SHAPES = [(1, 136, 256), (7, 136, 384), (33, 4104, 2048), (64, 264, 640), (100, 2112, 384),
          (128, 1000, 256), (64, 2112, 7168), (128, 4096, 1024), (50, 7168, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_cluster_split_each_size(fg, M, N, K):
    case = synth.dense_case(800 + M, M, N, K, row_scaled=True)
    case.update(M=M, N=N, K=K)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    tiles, kb = -(-N // 128), -(-K // 128)
    ran = set()
    for S in (2, 4, 8):
        plan, got = run(fg, case, S)
        assert plan == S or S > kb or plan in (0, 1), plan  # S, or a fallback when S cannot be resident
        ran.add(plan)
        close(got, ref, f"{M}x{N}x{K} schedule {S} (ran {plan})")
        if plan == S:  # bit-reproducible: partials summed in rank order
            np.testing.assert_array_equal(run(fg, case, S)[1], got)
    plan, got = run(fg, case, -1)
    assert plan in (0, 1)
    close(got, ref, f"{M}x{N}x{K} no cluster")
    if kb >= 2 and tiles <= 16:
        assert 2 in ran, "the two-CTA cluster split never ran"


@pytest.mark.parametrize("w", workloads.decode_sweep(), ids=lambda w: w["name"])
def test_decode_shapes_automatic_schedule(fg, w):
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"], row_scaled=True)
    case.update(M=w["M"], N=w["N"], K=w["K"])
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    plan, got = run(fg, case, 0)
    close(got, ref, f"{w['name']} automatic (schedule {plan})")


def test_cluster_timeout_path(fg):
    """The MMA thread of every CTA waits on a barrier no one arrives at; the bounded wait runs
    out, every thread still reaches both cluster barriers, the status word reads FG_ERR_TIMEOUT,
    and the next call gives the same bits as before."""
    case = synth.dense_case(871, 64, 2112, 2048, row_scaled=True)
    case.update(M=64, N=2112, K=2048)
    old = fg.set_swap_schedule(4)
    old_path = fg.set_dense_path(2)
    try:
        assert fg.swap_plan(64, 2112, 2048) == 4
        A, sfa, B, sfb = dense_dev(case)
        before = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
        torch.cuda.synchronize()
        assert fg.device_status() == 0
        stall = fg.lib.fg_debug_set_stall(1)
        try:
            t0 = time.time()
            fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
            status = fg.device_status()
            elapsed = time.time() - t0
        finally:
            fg.lib.fg_debug_set_stall(stall)
        assert status == FG_ERR_TIMEOUT, status
        assert 1.0 < elapsed < 20.0, elapsed
        after = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(after, before)
        assert fg.device_status() == 0
    finally:
        fg.set_swap_schedule(old)
        fg.set_dense_path(old_path)
