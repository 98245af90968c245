"""GPU parity: the CUDA path (through the C ABI binding) against the CPU oracle.

Every comparison uses the stated tolerance (tests/gpu_helpers.py):
elementwise |c - r| <= 0.01 |r| + 1e-3 max|r| and per matrix
1 - 2 sum(c r) / sum(c^2 + r^2) < 1e-5.  Every benchmark matrix (the pages' normal,
contiguous and masked tables) is checked whole, every row and column, in the launch
configuration the benchmark times; the prefill and contiguous matrices take the
oracle about two minutes on 16 host cores together.  The CTA-pair kernel is checked
on sampled prefill rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import bits_of, close, dense_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import moe_grouped_gemm_08_b200 as lib
    torch.cuda.set_device(0)
    lib.init(0)
    yield lib
    lib.set_dense_path(0)


def canary_like(shape):
    """bf16 tensor whose every element has the bit pattern 0xFFFF (a NaN nobody writes)."""
    return torch.full(shape, -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def run_dense(fg, case, path):
    old = fg.set_dense_path(path)
    try:
        A, sfa, B, sfb = dense_dev(case)
        C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
        torch.cuda.synchronize()
    finally:
        fg.set_dense_path(old)
    return bits_of(C)


def sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, M // 2, M - 129, M - 128, M - 1]
    rows = np.unique(np.concatenate([[r for r in fixed if 0 <= r < M], rng.integers(0, M, n)]))
    return rows.astype(np.int32)


# --------------------------------------------------------------------------- dense
@pytest.mark.parametrize("path", [1, 2])
def test_dense_single(fg, path):
    w = workloads.dense_single()[0]
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"])
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    close(run_dense(fg, case, path), ref, f"dense_single path={path}")


ODD = [(1, 8, 16), (7, 136, 272), (33, 4104, 2048), (64, 264, 640), (100, 2112, 384), (128, 1000, 256),
       (129, 520, 256), (200, 136, 1152), (300, 392, 128), (513, 2048, 3072)]


@pytest.mark.parametrize("M,N,K", ODD)
def test_dense_odd_shapes(fg, M, N, K):
    case = synth.dense_case(100 + M, M, N, K, row_scaled=True)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    for path in ([1, 2, 3] if M <= 128 else [1, 3]):  # 1 tiled, 2 swap-AB stream-K, 3 CTA pair
        close(run_dense(fg, case, path), ref, f"odd {M}x{N}x{K} path={path}")


@pytest.mark.parametrize("bn", [128, 192, 256])
@pytest.mark.parametrize("M,N,K", [(129, 520, 256), (300, 392, 1152), (513, 2048, 3072), (1000, 2112, 640)])
def test_tile_widths(fg, bn, M, N, K):
    """Every tile width of the tiled kernel (and 192 / 256 of the CTA pair), with the stream-K tail
    forced, against the oracle: ragged M and N tails, partial waves."""
    case = synth.dense_case(700 + M, M, N, K, row_scaled=True)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    old = fg.set_tile_n(bn)
    old_sk = fg.set_tiled_streamk(0)
    try:
        for path in ([1, 3] if bn != 128 else [1]):
            close(run_dense(fg, case, path), ref, f"{M}x{N}x{K} bn={bn} path={path}")
    finally:
        fg.set_tile_n(old)
        fg.set_tiled_streamk(old_sk)


@pytest.mark.parametrize("schedule", [0, -1, 1, 2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(64, 2112, 7168), (128, 7168, 2048), (32, 1032, 1408), (100, 4096, 640),
                                   (7, 264, 384)])
def test_swap_two_kblocks_per_stage(fg, schedule, M, N, K):
    """The small-M kernel with two K blocks per ring stage (3-D copies; the default when K is a
    multiple of 128) against the oracle on every schedule, odd K-block counts included (the last
    stage of a tile then holds one K block); with whole tiles, bit-identical to one K block per
    stage (the same fp32 operations in the same order)."""
    case = synth.dense_case(800 + M, M, N, K, row_scaled=True)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    old = fg.set_swap_schedule(schedule)
    try:
        fg.set_stage_kblocks(2)
        two = run_dense(fg, case, 2)
        fg.set_stage_kblocks(1)
        one = run_dense(fg, case, 2)
    finally:
        fg.set_stage_kblocks(0)
        fg.set_swap_schedule(old)
    close(two, ref, f"kps=2 {M}x{N}x{K} schedule {schedule}")
    close(one, ref, f"kps=1 {M}x{N}x{K} schedule {schedule}")
    if schedule == 1:
        np.testing.assert_array_equal(two, one)


@pytest.mark.parametrize("pw", [2, 4])
@pytest.mark.parametrize("M,N,K", [(300, 520, 1152), (513, 2048, 3072), (4096, 2112, 7168)])
def test_pair_kernel_promotion_warpgroups(fg, pw, M, N, K):
    """The 256-wide CTA-pair kernel with two and with four promotion warpgroups against the oracle
    (sampled rows for the large shape); both give the same bits (identical arithmetic)."""
    case = synth.dense_case(900 + M, M, N, K)
    rows = sample_rows(M, 40, M) if M > 1024 else None
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], rows=rows)
    old = (fg.set_tile_n(256), fg.set_pair_promotion(pw))
    try:
        got = run_dense(fg, case, 3)
        fg.set_pair_promotion(2 if pw == 4 else 4)
        other = run_dense(fg, case, 3)
    finally:
        fg.set_tile_n(old[0])
        fg.set_pair_promotion(old[1])
    close(got if rows is None else got[rows], ref, f"pair pw={pw} {M}x{N}x{K}")
    np.testing.assert_array_equal(got, other)


@pytest.mark.parametrize("w", workloads.decode_sweep(), ids=lambda w: w["name"])
def test_decode_sweep_full(fg, w):
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"], row_scaled=True)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    close(run_dense(fg, case, 0), ref, w["name"])
    if w["N"] * w["K"] <= 7168 * 7168:
        close(run_dense(fg, case, 1), ref, w["name"] + " tiled")


@pytest.mark.parametrize("w", workloads.prefill(), ids=lambda w: w["name"])
def test_prefill_full_matrix(fg, w):
    """The whole M=4096 output (every row and column) against the oracle, automatic kernel choice."""
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"])
    got = run_dense(fg, case, 0)
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"])
    close(got, ref, f"{w['name']} full")


@pytest.mark.parametrize("w", workloads.prefill(), ids=lambda w: w["name"])
def test_prefill_pair_kernel_sampled_rows(fg, w):
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"])
    rows = sample_rows(w["M"], 40, w["seed"])
    ref = oracle.gemm_nt(case["A"], case["sfa"], case["B"], case["sfb"], rows=rows)
    got = run_dense(fg, case, 3)  # the CTA-pair kernel
    close(got[rows], ref, f"{w['name']} path=3")


@pytest.mark.parametrize("idx", [0, 6, 8])
def test_stream_k_deterministic(fg, idx):
    """Split-K partials are summed in a fixed order: repeated calls are bit-identical."""
    w = workloads.decode_sweep()[idx]
    case = synth.dense_case(w["seed"], w["M"], w["N"], w["K"], row_scaled=True)
    a = run_dense(fg, case, 2)
    for _ in range(2):
        np.testing.assert_array_equal(run_dense(fg, case, 2), a)


def test_dense_m_zero_is_noop(fg):
    A = torch.zeros((0, 128), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((1, 0), dtype=torch.float32, device="cuda")
    B = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    sfb = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    C = fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb)
    assert C.shape == (0, 128)


# --------------------------------------------------------------------------- contiguous
def run_contig(fg, case, C=None):
    A, sfa = to_dev(case["A"]), to_dev(case["sfa"])
    B, sfb = to_dev(case["B"]), to_dev(case["sfb"])
    mi = to_dev(case["m_indices"])
    if C is None:
        C = canary_like((case["M"], case["N"]))
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(A, sfa, B, sfb, mi, C=C)
    torch.cuda.synchronize()
    return bits_of(C)


def test_contiguous_odd_padding(fg):
    case = synth.contiguous_case(41, [100, 0, 300, 37, 128, 1], N=264, K=384)
    got = run_contig(fg, case)
    canary = np.full((case["M"], case["N"]), 0xFFFF, dtype=np.uint16)
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"], C=canary)
    live = case["m_indices"] >= 0
    close(got[live], ref[live], "contiguous odd")
    assert np.all(got[~live] == 0xFFFF), "padding rows were written"


def test_contiguous_out_of_range_index_is_skipped(fg):
    case = synth.contiguous_case(42, [128, 128, 128], N=136, K=256)
    mi = case["m_indices"].copy()
    mi[256:384] = 7  # >= G: treated as padding
    case["m_indices"] = mi
    got = run_contig(fg, case)
    assert np.all(got[256:] == 0xFFFF)
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], mi)
    close(got[:256], ref[:256], "contiguous index >= G")


@pytest.mark.parametrize("w", workloads.contiguous(), ids=lambda w: w["name"])
def test_contiguous_full_matrix(fg, w):
    """The whole 32768-row output against the oracle: both criteria over the complete matrix, and
    each expert's block of rows on its own."""
    case = synth.contiguous_case(w["seed"], [w["M_per_group"]] * w["G"], w["N"], w["K"])
    got = run_contig(fg, case, C=torch.empty((case["M"], case["N"]), dtype=torch.bfloat16, device="cuda"))
    ref = oracle.grouped_contiguous(case["A"], case["sfa"], case["B"], case["sfb"], case["m_indices"])
    close(got, ref, f"{w['name']} full")
    Mg = w["M_per_group"]
    for g in range(w["G"]):
        close(got[g * Mg:(g + 1) * Mg], ref[g * Mg:(g + 1) * Mg], f"{w['name']} expert {g}")


# --------------------------------------------------------------------------- masked
def masked_dev(case):
    return (to_dev(case["A"]), to_dev(case["sfa"]), to_dev(case["B"]), to_dev(case["sfb"]),
            to_dev(case["masked_m"]))


def check_masked(got, case, what):
    G, Mmax, N = case["G"], case["Mmax"], case["N"]
    canary = np.full((G, Mmax, N), 0xFFFF, dtype=np.uint16)
    ref = oracle.grouped_masked(case["A"], case["sfa"], case["B"], case["sfb"], case["masked_m"], C=canary)
    for g in range(G):
        v = min(int(case["masked_m"][g]), Mmax)
        if v:
            close(got[g, :v], ref[g, :v], f"{what} g={g}")
        assert np.all(got[g, v:] == 0xFFFF), f"{what}: rows past masked_m[{g}]={v} were written"


@pytest.mark.parametrize("path", [0, 3], ids=["tiled", "pair"])
@pytest.mark.parametrize("w", workloads.masked(), ids=lambda w: w["name"])
def test_masked_under_cuda_graph(fg, w, path):
    old_path = fg.set_dense_path(path)  # the masked entry point takes the CTA-pair kernel with 3
    try:
        _masked_under_cuda_graph(fg, w)
    finally:
        fg.set_dense_path(old_path)


def _masked_under_cuda_graph(fg, w):
    case = synth.masked_case(w["seed"], w["G"], w["Mmax"], w["N"], w["K"])
    A, sfa, B, sfb, mm = masked_dev(case)
    C = canary_like((w["G"], w["Mmax"], w["N"]))
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)  # warm-up outside capture
    C.view(torch.int16).fill_(-1)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)
    C.view(torch.int16).fill_(-1)
    graph.replay()
    torch.cuda.synchronize()
    check_masked(bits_of(C), case, w["name"])
    # new counts written into the same device buffer, same graph replayed
    if w["G"] >= 2:
        new = np.array(case["masked_m"][::-1], dtype=np.int32)
        mm.copy_(torch.from_numpy(new).cuda())
        C.view(torch.int16).fill_(-1)
        graph.replay()
        torch.cuda.synchronize()
        case2 = dict(case, masked_m=new)
        check_masked(bits_of(C), case2, w["name"] + " replay")
    else:
        for cnt in (0, 333):
            mm.fill_(cnt)
            C.view(torch.int16).fill_(-1)
            graph.replay()
            torch.cuda.synchronize()
            check_masked(bits_of(C), dict(case, masked_m=np.array([cnt], np.int32)), f"{w['name']} m={cnt}")
    del graph


@pytest.mark.parametrize("path", [0, 3], ids=["tiled", "pair"])
def test_masked_counts_edge_cases(fg, path):
    old_path = fg.set_dense_path(path)
    try:
        _masked_counts_edge_cases(fg)
    finally:
        fg.set_dense_path(old_path)


def _masked_counts_edge_cases(fg):
    case = synth.masked_case(51, 3, 200, 136, 256, masked_m=[0, 0, 0])
    A, sfa, B, sfb, mm = masked_dev(case)
    C = canary_like((3, 200, 136))
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)
    torch.cuda.synchronize()
    assert np.all(bits_of(C) == 0xFFFF)
    mm.copy_(torch.tensor([500, 1, 129], dtype=torch.int32, device="cuda"))  # 500 > Mmax: clamped
    fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, mm, C=C)
    torch.cuda.synchronize()
    check_masked(bits_of(C), dict(case, masked_m=np.array([200, 1, 129], np.int32)), "masked edge")


def test_device_status_clean(fg):
    assert fg.device_status() == 0


def test_output_in_host_memory_is_rejected(fg):
    """A host-memory output is refused before any launch, for all three layouts."""
    case = synth.dense_case(7, 64, 256, 256)
    A, sfa, B, sfb = dense_dev(case)
    before = fg.launch_count()
    with pytest.raises(ValueError):
        fg.gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, C=torch.empty((64, 256), dtype=torch.bfloat16))
    cc = synth.contiguous_case(8, [64, 64], N=136, K=256)
    with pytest.raises(ValueError):
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(to_dev(cc["A"]), to_dev(cc["sfa"]), to_dev(cc["B"]),
                                                     to_dev(cc["sfb"]), to_dev(cc["m_indices"]),
                                                     C=torch.empty((cc["M"], cc["N"]), dtype=torch.bfloat16))
    mc = synth.masked_case(9, 2, 128, 136, 256, masked_m=[5, 128])
    with pytest.raises(ValueError):
        fg.m_grouped_gemm_fp8_fp8_bf16_nt_masked(to_dev(mc["A"]), to_dev(mc["sfa"]), to_dev(mc["B"]),
                                                 to_dev(mc["sfb"]), to_dev(mc["masked_m"]),
                                                 C=torch.empty((2, 128, 136), dtype=torch.bfloat16))
    assert fg.launch_count() == before
