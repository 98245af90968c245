#!/usr/bin/env python
"""Benchmark of the FP8 block-scaled NT GEMM on B200.

One step = one pass of the chosen workload (default: the dense decode sweep, M in
{64,128} x six (N,K) DeepSeek-V3/R1 shapes = 12 GEMM launches) over inputs
already resident in HBM.  Prints ONE JSON line on rank 0.  The headline keys
(value, roofline, e2e, cpu_baseline) are the decode sweep's; the other four
configurations (dense 128x256x512, prefill M=4096, contiguous, masked) are timed
the same way in the same run, with the same steps and warm-up, and reported under
"workloads" (--also selects them).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--also LIST]
                  [--impl ours|reference]

Timing: each step is replayed from a CUDA graph (the masked-layout call is made
for graphs; the dense calls are captured the same way so that host launch cost
does not hide in the device timeline).  Inputs rotate over R copies whose total
size is several times the 126 MB L2, so every launch reads its operands from HBM.
The timed region is bracketed by a barrier and torch.cuda.synchronize() on both
sides and measured with CUDA events on the launching stream; multi-GPU runs take
the max over ranks (independent replicas: the GEMM needs no exchange step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from synth import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense fp8 / bf16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)
KERNEL_SOURCES = ["moe_grouped_gemm_08_b200/csrc/fp8_gemm_kernels.cuh",
                  "moe_grouped_gemm_08_b200/csrc/fp8_cast_kernels.cuh",
                  "moe_grouped_gemm_08_b200/csrc/sm100_ptx.cuh",
                  "moe_grouped_gemm_08_b200/csrc/fp8gemm_api.cu"]


# ---------------------------------------------------------------------------- helpers
def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained") if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get(f"{kernel}:{workload}")
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash():
        return None
    return entry


def record_traffic(csv_path: str, workload: str, out_path: str | None = None) -> None:
    """Average dram__bytes_read.sum + dram__bytes_write.sum per launch of each of this library's
    kernels in an ncu --csv launch list, stored (default: profiles/traffic.json) with the kernel
    source hash."""
    import csv as _csv
    rows = [r for r in _csv.reader(open(csv_path)) if r]
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r and "Metric Name" in r)
    h = rows[hi]
    col = {k: h.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    per = {}
    for r in rows[hi + 1:]:
        if len(r) != len(h) or not r[col["Metric Name"]].startswith("dram__bytes_"):
            continue
        name = r[col["Kernel Name"]]
        kern = next((k for k in ("fp8_gemm_swap_streamk_kernel", "fp8_gemm_tiled_kernel", "fp8_gemm_pair_kernel")
                     if k in name), None)
        if kern is None:
            continue
        unit = r[col["Metric Unit"]]
        if unit not in scale:
            raise ValueError(f"unexpected unit {unit!r} for {r[col['Metric Name']]}")
        v = float(r[col["Metric Value"]].replace(",", "")) * scale[unit]
        per.setdefault(kern, {}).setdefault(r[col["ID"]], 0.0)
        per[kern][r[col["ID"]]] += v
    path = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    d = json.load(open(path)) if os.path.exists(path) else {}
    for kern, launches in per.items():
        d[f"{kern}:{workload}"] = {"dram_bytes_per_launch": round(sum(launches.values()) / len(launches)),
                                   "launches": len(launches), "kernel_source_hash": kernel_source_hash(),
                                   "source": os.path.basename(csv_path)}
    with open(path, "w") as f:
        json.dump(d, f, indent=1, sort_keys=True)
    print(json.dumps({k: v for k, v in d.items() if k.endswith(":" + workload)}))


def cdiv(a, b):
    return (a + b - 1) // b


def workload_list(name: str, shape: str | None = None):
    if shape:
        M, N, K = (int(x) for x in shape.split(","))
        return f"dense_M{M}_N{N}_K{K}", [dict(name=f"dense_M{M}_N{N}_K{K}", seed=77, M=M, N=N, K=K,
                                              row_scaled=M <= 128)]
    table = {"decode_sweep": workloads.decode_sweep, "dense_single": workloads.dense_single,
             "prefill": workloads.prefill, "contiguous": workloads.contiguous, "masked": workloads.masked}
    if name not in table:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(table)}")
    return name, table[name]()


def make_case(w):
    if "Mmax" in w:
        return synth.masked_case(w["seed"], w["G"], w["Mmax"], w["N"], w["K"])
    if "M_per_group" in w:
        return synth.contiguous_case(w["seed"], [w["M_per_group"]] * w["G"], w["N"], w["K"])
    return synth.dense_case(w["seed"], w["M"], w["N"], w["K"], row_scaled=w.get("row_scaled", False))


def work_of(case):
    """(flops, algorithmic bytes incl. scales, pages-style bytes A+B+C) of one call, valid rows only."""
    N, K = case["N"], case["K"]
    KB, NB = cdiv(K, 128), cdiv(N, 128)
    if case["kind"] == "masked":
        valid = np.clip(np.asarray(case["masked_m"], dtype=np.int64), 0, case["Mmax"])  # as the kernel reads it
        Mv = int(valid.sum())
        groups_used = int((valid > 0).sum())
        G = case["G"]
        flops = 2 * Mv * N * K
        byt = Mv * K + groups_used * N * K + 2 * Mv * N + 4 * Mv * KB + 4 * groups_used * NB * KB
        pages = G * case["Mmax"] * K + G * N * K + 2 * G * case["Mmax"] * N
        return flops, byt, pages
    if case["kind"] == "contiguous":
        mi = np.asarray(case["m_indices"])
        live = (mi >= 0) & (mi < case["G"])  # indices >= G are padding, as in the kernel
        Mv = int(live.sum())
        groups_used = int(np.unique(mi[live]).size)  # B is needed only for groups with a valid row
        flops = 2 * Mv * N * K
        byt = Mv * K + groups_used * N * K + 2 * Mv * N + 4 * Mv * KB + 4 * groups_used * NB * KB
        return flops, byt, Mv * K + groups_used * N * K + 2 * Mv * N
    M = case["M"]
    flops = 2 * M * N * K
    byt = M * K + N * K + 2 * M * N + 4 * M * KB + 4 * NB * KB
    return flops, byt, M * K + N * K + 2 * M * N


_FG = None  # the binding, once run_ours has loaded it


def kernel_name(case) -> str:
    """The library kernel a case runs on under the current settings (the library's own plan)."""
    if case["kind"] == "masked":
        plan = _FG.tile_plan("masked", case["Mmax"], case["N"], case["K"], case["G"])
    elif case["kind"] == "contiguous":
        plan = _FG.tile_plan("contiguous", case["M"], case["N"], case["K"], case["G"])
    else:
        plan = _FG.tile_plan("dense", case["M"], case["N"], case["K"], 1)
    return {1: "fp8_gemm_tiled_kernel", 2: "fp8_gemm_swap_streamk_kernel",
            3: "fp8_gemm_pair_kernel"}.get(plan // 1000, "unknown")


def tile_width(case):
    if case["kind"] == "dense" and case["M"] <= 128:
        return None
    layout = case["kind"]
    M = case["Mmax"] if layout == "masked" else case["M"]
    return _FG.tile_plan(layout, M, case["N"], case["K"], case.get("G", 1)) % 1000


def upload(case, dev):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    d = dict(A=t(case["A"]), sfa=t(case["sfa"]), B=t(case["B"]), sfb=t(case["sfb"]))
    if case["kind"] == "masked":
        d["masked_m"] = t(case["masked_m"])
        d["C"] = torch.empty((case["G"], case["Mmax"], case["N"]), dtype=torch.bfloat16, device=dev)
    elif case["kind"] == "contiguous":
        d["m_indices"] = t(case["m_indices"])
        d["C"] = torch.empty((case["M"], case["N"]), dtype=torch.bfloat16, device=dev)
    else:
        d["C"] = torch.empty((case["M"], case["N"]), dtype=torch.bfloat16, device=dev)
    return d


def call(fg, case, d, stream=None, static_b=False):
    if case["kind"] == "masked":
        return fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(d["A"], d["sfa"], d["B"], d["sfb"], d["masked_m"],
                                                        C=d["C"], stream=stream)
    if case["kind"] == "contiguous":
        return fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(d["A"], d["sfa"], d["B"], d["sfb"], d["m_indices"],
                                                            C=d["C"], stream=stream)
    return fg.gemm_fp8_fp8_bf16_nt(d["A"], d["sfa"], d["B"], d["sfb"], C=d["C"], stream=stream, static_b=static_b)


_CUDART = None


def record_event_node(ev: torch.cuda.Event, stream: torch.cuda.Stream) -> None:
    """Record `ev` on `stream` so that, during stream capture, it becomes an event-record node of the
    graph (cudaEventRecordExternal): its timestamp is then readable after every replay."""
    global _CUDART
    import ctypes
    if _CUDART is None:
        _CUDART = ctypes.CDLL("libcudart.so.12")
        _CUDART.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        _CUDART.cudaEventRecordWithFlags.restype = ctypes.c_int
    rc = _CUDART.cudaEventRecordWithFlags(ctypes.c_void_p(ev.cuda_event), ctypes.c_void_p(stream.cuda_stream), 1)
    if rc != 0:
        raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            # a timed region shorter than nvidia-smi's start-up would otherwise end with no sample
            deadline = time.time() + 3.0
            while not self.samples and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.02)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inside = [s for (ts, s) in self.samples if t0 - 0.05 <= ts <= t1 + 0.15]
        note = None
        if not inside:  # timed region shorter than the sampling period: nearest samples
            inside = [min(self.samples, key=lambda x: abs(x[0] - (t0 + t1) / 2))[1]]
            note = "timed region shorter than the 100 ms sampling period; nearest sample"
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(s[2]) for s in inside if num(s[2]) is not None]
        smax = [num(s[3]) for s in inside if num(s[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in inside for i in range(4) if len(s) > 6 + i and s[6 + i] == "Active"})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
               "reasons": reasons, "samples": len(inside)}
        if note:
            out["note"] = note
        return out


# ---------------------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- CPU oracle timing
def time_oracle(cases, row_fraction: float = 1.0):
    """Time the CPU oracle as it stands over (a row sample of) the cases; returns (seconds, flops, desc)."""
    import oracle  # the oracle is test infrastructure; only this leg of the benchmark runs it
    flops = 0
    t0 = time.perf_counter()
    for c in cases:
        if c["kind"] == "dense":
            M = c["M"]
            n = max(1, int(round(M * row_fraction)))
            rows = np.linspace(0, M - 1, n).astype(np.int32)
            oracle.gemm_nt(c["A"], c["sfa"], c["B"], c["sfb"], rows=rows if n < M else None)
            flops += 2 * n * c["N"] * c["K"]
        elif c["kind"] == "contiguous":
            M = c["M"]
            n = max(1, int(round(M * row_fraction)))
            rows = np.linspace(0, M - 1, n).astype(np.int32)
            oracle.grouped_contiguous(c["A"], c["sfa"], c["B"], c["sfb"], c["m_indices"], rows=rows)
            flops += 2 * int((c["m_indices"][rows] >= 0).sum()) * c["N"] * c["K"]
        else:
            mm = np.minimum(c["masked_m"], c["Mmax"])
            sub = np.maximum(1, np.round(mm * row_fraction)).astype(np.int32) * (mm > 0)
            oracle.grouped_masked(c["A"], c["sfa"], c["B"], c["sfb"], sub)
            flops += 2 * int(sub.sum()) * c["N"] * c["K"]
    return time.perf_counter() - t0, flops, oracle.num_threads()


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the same workload, rank 0 only."""
    if rank != 0:
        return
    name, wl = workload_list(args.workload, args.shape)
    cases = [make_case(w) for w in wl]
    full_flops = sum(work_of(c)[0] for c in cases)
    # size each step so that warm-up + timed steps stay within about two minutes
    probe_s, probe_flops, cores = time_oracle(cases, row_fraction=min(1.0, 0.05))
    rate = probe_flops / max(probe_s, 1e-9)
    budget_per_step = 120.0 / max(1, args.steps + args.warmup)
    frac = float(min(1.0, max(1e-4, budget_per_step * rate / full_flops)))
    for _ in range(args.warmup):
        time_oracle(cases, frac)
    total_s, total_flops = 0.0, 0
    for _ in range(args.steps):
        s, f, cores = time_oracle(cases, frac)
        total_s += s
        total_flops += f
    value = total_flops / total_s / 1e12
    sample = f"{frac:.4g} of the rows of every GEMM of the {name} workload per step (evenly spaced rows)"
    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "shapes": [w["name"] for w in wl]}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


METRIC = "FP8 TFLOPS & HBM GB/s per GEMM shape on 1xB200; % of FP8/HBM roofline"


# ---------------------------------------------------------------------------- the cast step
def run_cast(args, rank, world, local):
    """Time the cast step (bf16 -> e4m3 + fp32 scales) on the prefill workload's operands: the
    activations [4096, K] (1x128 row scales) and the weights [N, K] (128x128 block scales) of its
    six GEMMs, 12 launches per step; about 1.1 GB moved per step, over 3x L2."""
    import moe_grouped_gemm_08_b200 as fg
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = workloads.prefill()
    g = torch.Generator(device=dev).manual_seed(5)
    xs = [torch.randn((w["M"], w["K"]), generator=g, device=dev).to(torch.bfloat16) for w in wl]
    ws = [torch.randn((w["N"], w["K"]), generator=g, device=dev).to(torch.bfloat16) for w in wl]
    outs = [fg.cast_fp8_rows(x) for x in xs] + [fg.cast_fp8_blocks(w) for w in ws]

    def launch_all():
        s = torch.cuda.current_stream()
        for x, (q, sfa) in zip(xs, outs[:len(xs)]):
            fg._check(fg.lib.fp8_cast_rows(x.data_ptr(), q.data_ptr(), sfa.data_ptr(), 1, x.shape[0], x.shape[1],
                                           fg._stream(s)), "cast rows")
        for w, (q, sfb) in zip(ws, outs[len(xs):]):
            fg._check(fg.lib.fp8_cast_blocks(w.data_ptr(), q.data_ptr(), sfb.data_ptr(), 1, w.shape[0], w.shape[1],
                                             fg._stream(s)), "cast blocks")

    def nbytes(M, K, rows):
        kb = cdiv(K, 128)
        return 3 * M * K + 4 * (M * kb if rows else cdiv(M, 128) * kb)
    step_bytes = sum(nbytes(x.shape[0], x.shape[1], True) for x in xs) + \
        sum(nbytes(w.shape[0], w.shape[1], False) for w in ws)
    graph = torch.cuda.CUDAGraph()
    launch_all()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        launch_all()
    for _ in range(args.warmup):
        graph.replay()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world, local)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record()
    for _ in range(args.steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world, local)
    clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    gbs = step_bytes * args.steps * world / (ms * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    del graph
    if rank == 0:
        line = {"metric": "HBM GB/s of the FP8 cast (bf16 -> e4m3 codes + fp32 scales)", "value": round(gbs, 1),
                "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 -> e4m3", "data": "synthetic",
                "config": {"workload": "cast_prefill_operands", "launches_per_step": 12,
                           "bytes_per_step": step_bytes, "graph": "each step replayed from a CUDA graph"},
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None,
                             "peak_source": f"{peak_src} (hbm_gbs)",
                             "bytes_per_launch_def": "2 bytes read + 1 byte written per element + fp32 scales"},
                "gpu_launches": 12 * args.steps, "clocks": clocks.summary(t0, t1)}
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- our arm
def measure_workload(fg, name, wl, args, dev, stream, world, local, static_b=False):
    """Time one workload: each step (one call per GEMM of the workload) is replayed from a CUDA
    graph, inputs rotating over enough copies that every launch reads HBM.  Returns the workload's
    result dict, its cases and the device copies (for the end-to-end leg)."""
    cases = [make_case(w) for w in wl]
    works = [work_of(c) for c in cases]
    step_flops = sum(w[0] for w in works)
    step_bytes = sum(w[1] for w in works)
    step_in_bytes = sum(c["A"].nbytes + c["B"].nbytes + c["sfa"].nbytes + c["sfb"].nbytes for c in cases)

    # rotation: enough input copies that one copy is re-read only after > 3x L2 of other traffic
    rot = max(2, min(8, cdiv(3 * L2_BYTES, max(1, step_in_bytes)) + 1))
    devs = [[upload(c, dev) for c in cases] for _ in range(rot)]

    # eager warm-up call per case (sets kernel attributes before capture), then capture one graph per copy
    with torch.cuda.stream(stream):
        for c, d in zip(cases, devs[0]):
            call(fg, c, d, stream=stream, static_b=static_b)
    stream.synchronize()
    launches_before = fg.launch_count()
    graphs = []       # kernels only: the timed region (consecutive launches may overlap via PDL)
    for r in range(rot):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c, d in zip(cases, devs[r]):
                call(fg, c, d, stream=stream, static_b=static_b)
        graphs.append(g)
    launches_per_step = (fg.launch_count() - launches_before) // rot
    egraphs, gevents = [], []  # the same step with an event node around every launch: per-shape times
    for r in range(rot):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(cases) + 1)]
        for ev in evs:  # create the CUDA events outside capture
            ev.record(stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i, (c, d) in enumerate(zip(cases, devs[r])):
                record_event_node(evs[i], stream)
                call(fg, c, d, stream=stream, static_b=static_b)
            record_event_node(evs[-1], stream)
        egraphs.append(g)
        gevents.append(evs)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for k in range(args.warmup):
        graphs[k % rot].replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record(stream)
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            graphs[(args.warmup + k) % rot].replay()
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world, local)
    time.sleep(0.25)
    clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    # per-shape device durations: a separate pass over the event-instrumented graphs
    per_case_ms = [[] for _ in cases]
    with torch.cuda.stream(stream):
        for k in range(3 * rot):
            egraphs[k % rot].replay()
            stream.synchronize()
            evs = gevents[k % rot]
            for i in range(len(cases)):
                per_case_ms[i].append(evs[i].elapsed_time(evs[i + 1]))
    status = fg.device_status(stream)
    del graphs, egraphs

    total_flops = step_flops * args.steps * world
    value = total_flops / (elapsed_ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    shapes = []
    sum_bytes_dom, sum_ms_dom, sum_ms_all = 0.0, 0.0, 0.0
    # the dominant kernel: the one with the largest share of the event-timed launch durations
    share = {}
    for c, ts in zip(cases, per_case_ms):
        share[kernel_name(c)] = share.get(kernel_name(c), 0.0) + statistics.mean(ts)
    dom = max(share, key=share.get)
    for c, w, wk, ts in zip(cases, wl, works, per_case_ms):
        ms = statistics.mean(ts)
        tfl = wk[0] / (ms * 1e-3) / 1e12
        gbs = wk[1] / (ms * 1e-3) / 1e9
        t_roof = max(wk[0] / (fp8_peak * 1e12), wk[1] / (peaks["hbm_gbs"] * 1e9))
        shapes.append({"name": w["name"], "us": round(ms * 1e3, 2), "tflops": round(tfl, 1), "gbs": round(gbs, 1),
                       "pages_gbs": round(wk[2] / (ms * 1e-3) / 1e9, 1),
                       "bound": "hbm" if wk[1] / (peaks["hbm_gbs"] * 1e9) > wk[0] / (fp8_peak * 1e12) else "tensor",
                       "roofline_frac": round(t_roof / (ms * 1e-3), 3), "kernel": kernel_name(c)})
        if kernel_name(c) == "fp8_gemm_swap_streamk_kernel":
            plan = fg.swap_plan(c["M"], c["N"], c["K"])
            shapes[-1]["schedule"] = {0: "stream-K", 1: "whole tiles"}.get(plan, f"cluster x{plan}")
        else:
            shapes[-1]["tile_n"] = tile_width(c)
        sum_ms_all += ms
        if kernel_name(c) == dom:
            sum_bytes_dom += wk[1]
            sum_ms_dom += ms
    # the roofline's bound is the one of the dominant kernel's work taken together
    dom_flops = sum(wk[0] for c, wk in zip(cases, works) if kernel_name(c) == dom)
    dom_bound = "hbm" if sum_bytes_dom / (peaks["hbm_gbs"] * 1e9) > dom_flops / (fp8_peak * 1e12) else "tensor"
    single_kernel = all(kernel_name(c) == dom for c in cases)
    if single_kernel:
        # every launch of the timed region is this kernel: its average launch duration is the
        # timed region divided by the launches (inter-kernel gaps included)
        sum_ms_dom = elapsed_ms / args.steps
        sum_ms_all = sum_ms_dom
    if dom_bound == "hbm":
        achieved = sum_bytes_dom / (sum_ms_dom * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4)}
    else:
        achieved = dom_flops / (sum_ms_dom * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / fp8_peak, 4)}
    tr = load_traffic(dom, name)
    roof["traffic"] = tr["dram_bytes_per_launch"] if tr else None
    roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if dom_bound == 'hbm' else 'bf16_tflops x 2 nominal fp8/bf16'})"
    roof["kernel"] = dom
    roof["launch_share"] = round(sum_ms_dom / sum_ms_all, 4) if sum_ms_all else None
    roof["algorithmic_bytes_per_step"] = int(sum_bytes_dom)
    roof["algorithmic_flops_per_step"] = int(dom_flops)
    roof["bytes_per_launch_def"] = "A + B + C + fp32 scales, valid rows, per launch; summed over the step"
    roof["timing"] = ("timed region / launches" if single_kernel else
                      "event-instrumented pass after the timed region")
    res = {"value": round(value, 2), "unit": "TFLOPS", "ms_per_step": round(elapsed_ms / args.steps, 5),
           "steps": args.steps, "warmup": args.warmup,
           "hbm_gbs": round(step_bytes * args.steps * world / (elapsed_ms * 1e-3) / 1e9, 1),
           "config": {"workload": name, "shapes": [w["name"] for w in wl],
                      "l2": f"inputs rotate over {rot} copies ({rot * step_in_bytes / 1e6:.0f} MB > L2)",
                      "graph": "each step replayed from a CUDA graph",
                      "static_b": static_b},
           "shapes": shapes, "shapes_timing": "event node around each launch, separate pass after the timed region",
           "roofline": roof, "gpu_launches": launches_per_step * args.steps,
           "clocks": clocks.summary(t_wall0, t_wall1), "device_status": fg.STATUS_NAMES.get(status, status)}
    return res, cases, devs, step_flops


def box_copy_gbs(dev) -> float:
    """This GPU's copy bandwidth now (read + write bytes of a 1 GiB bf16 copy, best of 5, CUDA events):
    context for comparing runs on different machines; the roofline uses the measured peak."""
    a = torch.empty(1 << 29, dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    best = float("inf")
    for _ in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        b.copy_(a)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    torch.cuda.empty_cache()
    return round(2 * (1 << 30) / (best * 1e-3) / 1e9, 1)


def run_ours(args, rank, world, local):
    import moe_grouped_gemm_08_b200 as fg

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fg.init(local)
    global _FG
    _FG = fg
    fg.set_dense_path(args.path)
    if args.tiled_streamk is not None:
        fg.set_tiled_streamk(args.tiled_streamk)
    if args.swap_schedule is not None:
        fg.set_swap_schedule(args.swap_schedule)
    if args.tile_n is not None:
        fg.set_tile_n(args.tile_n)
    if args.stage_kblocks is not None:
        fg.set_stage_kblocks(args.stage_kblocks)
    if args.tile_order is not None:
        fg.set_tile_order(args.tile_order)
    stream = torch.cuda.Stream(device=dev)
    copy_gbs = box_copy_gbs(dev)
    name, wl = workload_list(args.workload, args.shape)
    # The weights of a decode step are loaded once and never rewritten, so the dense calls declare
    # them static (FG_FLAG_STATIC_B: weight tiles may load before the preceding launch ends);
    # --no-static-b times the fully stream-ordered form, which is also reported under "workloads".
    res, cases, devs, step_flops = measure_workload(fg, name, wl, args, dev, stream, world, local,
                                                    static_b=args.static_b)

    # end to end through the public API with host buffers: H2D of the step's inputs, GEMMs, D2H of C
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    host = []
    for c in cases:
        h = {k: torch.from_numpy(np.ascontiguousarray(c[k])).pin_memory() for k in ("A", "sfa", "B", "sfb")}
        if c["kind"] == "masked":
            h["masked_m"] = torch.from_numpy(c["masked_m"]).pin_memory()
        if c["kind"] == "contiguous":
            h["m_indices"] = torch.from_numpy(c["m_indices"]).pin_memory()
        host.append(h)
    outs = [torch.empty(tuple(devs[0][i]["C"].shape), dtype=torch.bfloat16).pin_memory() for i in range(len(cases))]
    h2d = sum(sum(t.numel() * t.element_size() for t in h.values()) for h in host)
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def e2e_step():
        for c, h, d, o in zip(cases, host, devs[0], outs):
            for key, t in h.items():
                d[key].copy_(t, non_blocking=True)
            call(fg, c, d, stream=stream)  # B is copied in just before: not static here
            o.copy_(d["C"], non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    barrier(world, local)
    e2e_value = step_flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12
    del host, outs, devs

    line = {"metric": METRIC, "value": res["value"], "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate, bf16 out)",
            "data": "synthetic",
            "config": dict(res["config"], parallelism=f"replicas x{world}", kernel_path=args.path,
                           tiled_streamk="library default" if args.tiled_streamk is None else args.tiled_streamk,
                           swap_schedule="library default" if args.swap_schedule is None else args.swap_schedule,
                           tile_n="library default" if args.tile_n is None else args.tile_n,
                           stage_kblocks="library default" if args.stage_kblocks is None else args.stage_kblocks,
                           tile_order="library default" if args.tile_order is None else args.tile_order),
            "hbm_gbs": res["hbm_gbs"], "shapes": res["shapes"], "shapes_timing": res["shapes_timing"],
            "roofline": res["roofline"],
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": res["gpu_launches"], "clocks": res["clocks"], "device_status": res["device_status"],
            "box_copy_gbs": copy_gbs}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        s, f, cores = time_oracle(cases, row_fraction=1.0)
        line["cpu_baseline"] = {"value": round(f / s / 1e12, 5), "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                "sample": f"one full step of the {name} workload (every GEMM, all rows), {s:.1f} s"}
    has_dense = any(c["kind"] == "dense" for c in cases)
    del cases
    torch.cuda.empty_cache()

    # the other configurations, timed the same way in the same process (same steps and warm-up)
    extra = [x for x in (args.also.split(",") if args.also else []) if x and x != name]
    if args.static_b and not args.shape and has_dense:
        extra = [name + ":ordered"] + extra
    if extra and not args.shape:
        line["workloads"] = {}
        for other in extra:
            base, _, mode = other.partition(":")
            oname, owl = workload_list(base)
            ores, ocases, odevs, _ = measure_workload(fg, oname, owl, args, dev, stream, world, local,
                                                      static_b=args.static_b and mode != "ordered")
            del ocases, odevs
            torch.cuda.empty_cache()
            line["workloads"][oname + (" (stream-ordered weights)" if mode == "ordered" else "")] = ores
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default="decode_sweep",
                    help="decode_sweep (default), dense_single, prefill, contiguous, masked, or cast (the bf16 -> "
                         "e4m3 cast of the prefill operands)")
    ap.add_argument("--shape", default=None, help="M,N,K: one dense GEMM instead of a workload (profiling)")
    ap.add_argument("--also", default="dense_single,prefill,contiguous,masked",
                    help="comma-separated workloads timed after the headline one in the same run, reported "
                         "under the 'workloads' key (empty: none)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-static-b", dest="static_b", action="store_false",
                    help="do not declare the weights static (FG_FLAG_STATIC_B) in the timed dense calls")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="kernel selection (fg_set_dense_path): 0 automatic, 1 one-CTA tiled, "
                         "2 swap-AB stream-K, 3 CTA pair")
    ap.add_argument("--tiled-streamk", type=int, default=None, metavar="BLOCKS",
                    help="tiled kernel's stream-K tail threshold (fg_set_tiled_streamk): split the last "
                         "partial wave when it saves more than BLOCKS K blocks; negative: never")
    ap.add_argument("--swap-schedule", type=int, default=None, choices=[-1, 0, 1, 2, 4, 8],
                    help="small-M kernel schedule (fg_set_swap_schedule): 0 automatic, -1 never the "
                         "cluster split, 1 whole tiles, 2/4/8 the cluster split with that many CTAs per tile")
    ap.add_argument("--tile-n", type=int, default=None, choices=[0, 128, 192, 256],
                    help="output tile width of the tiled / CTA-pair kernels (fg_set_tile_n): 0 automatic")
    ap.add_argument("--stage-kblocks", type=int, default=None, choices=[0, 1, 2],
                    help="K blocks per ring stage of the small-M and CTA-pair kernels (fg_set_stage_kblocks): "
                         "0 automatic")
    ap.add_argument("--tile-order", type=int, default=None, choices=[0, 1, 2],
                    help="tile walk of the tiled family (fg_set_tile_order): 0 automatic, 1 m-block groups, "
                         "2 n fastest")
    ap.add_argument("--record-traffic", default=None, metavar="CSV",
                    help="write profiles/traffic.json from an ncu launch list of this workload, then exit")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic, workload_list(args.workload, args.shape)[0])
        return
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload == "cast":
            run_cast(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
