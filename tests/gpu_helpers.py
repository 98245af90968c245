"""Shared helpers of the GPU parity tests: upload a synthetic case, call the CUDA path
through the binding, and compare with the oracle under the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances: elementwise |c - r| <= REL * |r| + ABS_OF_MAX * max|r|,
# and per matrix 1 - 2*sum(c*r) / sum(c^2 + r^2) < MATRIX.
REL = 0.01
ABS_OF_MAX = 1e-3
MATRIX = 1e-5


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bits_of(C: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return C.view(torch.int16).cpu().numpy().view(np.uint16)


def close(c_bits: np.ndarray, r_bits: np.ndarray, what: str = "") -> dict:
    """Check the two criteria; return the statistics, raise AssertionError on failure."""
    c = oracle.bf16_bits_to_f32(c_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(r_bits).astype(np.float64)
    assert c.shape == r.shape, (c.shape, r.shape)
    assert np.all(np.isfinite(r)), f"{what}: oracle produced non-finite values"
    if not np.all(np.isfinite(c)):
        bad = np.argwhere(~np.isfinite(c))[:5]
        raise AssertionError(f"{what}: non-finite GPU outputs at {bad.tolist()}")
    maxr = float(np.max(np.abs(r))) if r.size else 0.0
    err = np.abs(c - r)
    bound = REL * np.abs(r) + ABS_OF_MAX * maxr
    viol = err > bound
    denom = float(np.sum(c * c + r * r))
    diff = 1.0 - 2.0 * float(np.sum(c * r)) / denom if denom > 0 else 0.0
    stats = dict(max_abs_err=float(err.max()) if err.size else 0.0, max_ref=maxr, matrix_diff=diff,
                 violations=int(viol.sum()), exact_frac=float(np.mean(c_bits == r_bits)) if c.size else 1.0)
    if viol.any():
        idx = np.argwhere(viol)[:5]
        raise AssertionError(f"{what}: {int(viol.sum())} elements out of tolerance, e.g. at {idx.tolist()} "
                             f"gpu={c[tuple(idx[0])]} ref={r[tuple(idx[0])]} stats={stats}")
    assert diff < MATRIX, f"{what}: matrix-level difference {diff} >= {MATRIX} ({stats})"
    return stats


def dense_dev(case):
    return (to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]), to_dev(case["sfb"]))


def close_nonfinite(c_bits: np.ndarray, r_bits: np.ndarray, what: str = "") -> dict:
    """For outputs that non-finite input codes reach: NaN exactly where the oracle has NaN, the same
    signed infinity where it has one, and the finite rest within the stated tolerance."""
    c = oracle.bf16_bits_to_f32(c_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(r_bits).astype(np.float64)
    assert c.shape == r.shape, (c.shape, r.shape)
    nan_c, nan_r = np.isnan(c), np.isnan(r)
    if not np.array_equal(nan_c, nan_r):
        bad = np.argwhere(nan_c != nan_r)[:5]
        raise AssertionError(f"{what}: NaN positions differ, e.g. at {bad.tolist()}")
    inf_r = np.isinf(r)
    if not np.array_equal(np.isinf(c), inf_r) or not np.array_equal(c[inf_r], r[inf_r]):
        bad = np.argwhere((np.isinf(c) != inf_r) | (inf_r & (c != r)))[:5]
        raise AssertionError(f"{what}: infinities differ, e.g. at {bad.tolist()}")
    fin = ~(nan_r | inf_r)
    stats = close(c_bits[fin], r_bits[fin], what) if fin.any() else {}
    return dict(stats, nan=int(nan_r.sum()), inf=int(inf_r.sum()))
