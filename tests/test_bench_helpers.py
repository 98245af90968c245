"""CPU pins of the benchmark's measurement helpers: the algorithmic FLOPs and bytes per call (the
numerator of every roofline fraction), the ncu launch-list parser that records DRAM traffic, and
the clock-sample summary.  Expected values are written out from the definitions: FLOPs =
2 * valid rows * N * K; bytes = A and C of the valid rows + B of every group with a valid row +
fp32 scales (4 bytes per row per K block for A, per 128 x 128 block for B)."""
from __future__ import annotations

import csv
import json

import numpy as np
import pytest

import bench
import synth


def test_dense_work():
    c = dict(kind="dense", M=64, N=2112, K=7168)
    flops, byt, pages = bench.work_of(c)
    KB, NB = 56, 17
    assert flops == 2 * 64 * 2112 * 7168
    assert byt == 64 * 7168 + 2112 * 7168 + 2 * 64 * 2112 + 4 * 64 * KB + 4 * NB * KB
    assert pages == 64 * 7168 + 2112 * 7168 + 2 * 64 * 2112


def test_contiguous_work_counts_only_valid_rows_and_used_groups():
    c = synth.contiguous_case(1, [100, 0, 30], N=136, K=256)
    mi = c["m_indices"].copy()
    mi[5] = 7                      # an index >= G is padding as well
    c["m_indices"] = mi
    flops, byt, _ = bench.work_of(c)
    rows = 100 + 30 - 1            # group 1 is empty, one row of group 0 turned into padding
    assert flops == 2 * rows * 136 * 256
    groups = 2                     # groups 0 and 2 have valid rows; group 1's B is never read
    assert byt == rows * 256 + groups * 136 * 256 + 2 * rows * 136 + 4 * rows * 2 + 4 * groups * 2 * 2


def test_masked_work_clamps_counts_like_the_kernel():
    c = dict(kind="masked", G=3, Mmax=64, N=136, K=256, masked_m=np.array([-5, 80, 10], dtype=np.int32))
    flops, byt, pages = bench.work_of(c)
    rows = 0 + 64 + 10             # negative -> 0, above Mmax -> Mmax
    assert flops == 2 * rows * 136 * 256
    assert byt == rows * 256 + 2 * 136 * 256 + 2 * rows * 136 + 4 * rows * 2 + 4 * 2 * 2 * 2
    assert pages == 3 * 64 * 256 + 3 * 136 * 256 + 2 * 3 * 64 * 136   # the pages count full groups


def _ncu_csv(path, rows):
    hdr = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream", "Block Size",
           "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit", "Metric Value"]
    with open(path, "w", newline="") as f:
        f.write("==PROF== Connected to process 1\n")
        w = csv.writer(f, quoting=csv.QUOTE_ALL)
        w.writerow(hdr)
        for i, kern, metric, unit, value in rows:
            w.writerow([i, 1, "python", "h", kern, 1, 7, "(320, 1, 1)", "(148, 1, 1)", 0, "10.0",
                        "Command line profiler metrics", metric, unit, value])


def test_record_traffic_averages_read_plus_write_per_launch(tmp_path):
    k = "void fg::fp8_gemm_swap_streamk_kernel<64, 8>(CUtensorMap_st, CUtensorMap_st, fg::SwapParams)"
    t = "void fg::fp8_gemm_tiled_kernel<192, 4, 0>(CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, fg::TiledParams)"
    src = tmp_path / "launches.csv"
    _ncu_csv(src, [
        (0, k, "dram__bytes_read.sum", "Mbyte", "15.5"),
        (0, k, "dram__bytes_write.sum", "Kbyte", "500"),
        (0, k, "gpu__time_duration.sum", "us", "14.8"),          # not a DRAM metric: ignored
        (1, k, "dram__bytes_read.sum", "byte", "1,000,000"),      # thousands separators
        (1, k, "dram__bytes_write.sum", "byte", "0"),
        (2, t, "dram__bytes_read.sum", "Gbyte", "1.25"),
        (2, t, "dram__bytes_write.sum", "Mbyte", "250"),
    ])
    out = tmp_path / "traffic.json"
    bench.record_traffic(str(src), "demo", out_path=str(out))
    d = json.load(open(out))
    swap = d["fp8_gemm_swap_streamk_kernel:demo"]
    assert swap["launches"] == 2
    assert swap["dram_bytes_per_launch"] == round(((15.5e6 + 500e3) + 1e6) / 2)
    assert swap["kernel_source_hash"] == bench.kernel_source_hash()
    tiled = d["fp8_gemm_tiled_kernel:demo"]
    assert tiled["launches"] == 1 and tiled["dram_bytes_per_launch"] == round(1.25e9 + 250e6)


def test_record_traffic_rejects_an_unknown_unit(tmp_path):
    k = "void fg::fp8_gemm_tiled_kernel<192, 4, 0>(...)"
    src = tmp_path / "launches.csv"
    _ncu_csv(src, [(0, k, "dram__bytes_read.sum", "sector", "12")])
    with pytest.raises(ValueError, match="unexpected unit"):
        bench.record_traffic(str(src), "demo", out_path=str(tmp_path / "traffic.json"))


def test_clock_summary_median_max_and_reasons():
    s = bench.ClockSampler(0)
    fields = lambda sm, pc: ["0", "x", str(sm), "1965", "900", "x", "Not Active", "Not Active", "Not Active", pc]  # noqa: E731
    s.samples = [(10.00, fields(1900, "Not Active")), (10.10, fields(1965, "Active")), (10.20, fields(1800, "Not Active")),
                 (99.0, fields(100, "Not Active"))]  # the last one is outside the timed region
    out = s.summary(10.0, 10.2)
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
    empty = bench.ClockSampler(0).summary(0.0, 1.0)
    assert empty["sm_mhz"] is None and empty["samples"] == 0
