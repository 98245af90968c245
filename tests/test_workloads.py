"""The synthetic workloads use exactly the benchmark shapes of the product page's three tables
(tests/golden/benchmark_shapes.txt, cited there), in the same order, each once (CPU)."""
from __future__ import annotations

import os

from synth import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "benchmark_shapes.txt")


def golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            kind, G, M, N, K = line.split()
            rows.append((kind, int(G), int(M), int(N), int(K)))
    return rows


def test_dense_workloads_are_the_pages_normal_gemm_table():
    want = [r for r in golden_rows() if r[0] == "dense"]
    got = [("dense", 1, w["M"], w["N"], w["K"]) for w in workloads.decode_sweep() + workloads.prefill()]
    assert got == want


def test_grouped_workloads_are_the_pages_grouped_tables():
    rows = golden_rows()
    got = [("contiguous", w["G"], w["M_per_group"], w["N"], w["K"]) for w in workloads.contiguous()]
    assert got == [r for r in rows if r[0] == "contiguous"]
    got = [("masked", w["G"], w["Mmax"], w["N"], w["K"]) for w in workloads.masked()]
    assert got == [r for r in rows if r[0] == "masked"]


def test_seeds_are_distinct():
    seeds = [w["seed"] for f in (workloads.dense_single, workloads.decode_sweep, workloads.prefill,
                                 workloads.contiguous, workloads.masked) for w in f()]
    assert len(seeds) == len(set(seeds))
