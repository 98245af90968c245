"""CPU checks of the Python binding's operand checks: every operand and the output must live on
the GPU the launch goes to, and a given stream must belong to it (a pointer into host memory or
into another GPU would otherwise be dereferenced by the kernel).  The helpers compare devices
only, so they are checked here with host tensors and stand-in devices; no kernel is launched."""
from __future__ import annotations

import types

import pytest
import torch

import moe_grouped_gemm_08_b200 as fg

GPU0 = torch.device("cuda", 0)


def test_output_on_the_host_is_rejected():
    C = torch.empty((4, 8), dtype=torch.bfloat16)  # host memory
    with pytest.raises(ValueError, match="C is on cpu"):
        fg._out(C, (4, 8), GPU0)


def test_output_shape_and_dtype_are_checked_first():
    with pytest.raises(ValueError, match="shape"):
        fg._out(torch.empty((4, 9), dtype=torch.bfloat16), (4, 8), GPU0)
    with pytest.raises(ValueError, match="bfloat16"):
        fg._out(torch.empty((4, 8), dtype=torch.float32), (4, 8), GPU0)


def test_operands_on_another_device_are_rejected():
    with pytest.raises(ValueError, match="sfb is on cpu"):
        fg._same_device(GPU0, sfb=torch.zeros(2))
    fg._same_device(torch.device("cpu"), B=torch.zeros(2), sfa=torch.zeros(2))  # all on one device


def test_stream_of_another_device_is_rejected():
    other = types.SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=0)
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        fg._stream(other, GPU0)
    same = types.SimpleNamespace(device=GPU0, cuda_stream=1234)
    assert fg._stream(same, GPU0).value == 1234
