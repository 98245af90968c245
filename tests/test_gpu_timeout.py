"""The timeout path on the GPU, without a fault: the small-M dense kernel's MMA thread is made to
wait on a barrier that no one arrives at (fg_debug_set_stall).  The bounded wait runs out after
about two seconds, the kernel aborts cleanly and reports FG_ERR_TIMEOUT through the device status
word; the context stays usable and the next call gives the same bits as before."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import synth
from tests.gpu_helpers import bits_of, dense_dev

pytestmark = pytest.mark.gpu

FG_ERR_TIMEOUT = 6


def test_stalled_wait_reports_timeout_and_context_recovers():
    import moe_grouped_gemm_08_b200 as fg
    torch.cuda.set_device(0)
    fg.init(0)
    assert fg.device_status() == 0
    # 48 K blocks per CTA (more than the ring holds), so the abort cuts the work short
    case = synth.dense_case(61, 64, 7168, 16384, row_scaled=True)
    A, sfa, B, sfb = dense_dev(case)
    before = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
    torch.cuda.synchronize()

    old = fg.lib.fg_debug_set_stall(1)
    try:
        t0 = time.time()
        fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)  # the launch itself succeeds
        status = fg.device_status()              # synchronises, reads and clears the word
        elapsed = time.time() - t0
    finally:
        fg.lib.fg_debug_set_stall(old)
    assert status == FG_ERR_TIMEOUT, fg.STATUS_NAMES.get(status, status)
    assert 1.0 < elapsed < 20.0, elapsed                 # the ~2 s limit, not a hang
    assert fg.device_status() == 0                        # cleared by the read

    after = bits_of(fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(after, before)
    assert fg.device_status() == 0
