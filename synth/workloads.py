"""The synthetic workloads: shapes, seeds and value recipes (no GEMM arithmetic).

The shapes are the pages' benchmark shapes (the "DeepGEMM" product page,
flashmla.org, performance tables for normal, contiguous-grouped and
masked-grouped GEMMs: DeepSeek-V3/R1 layer shapes); the values are synthetic.

  dense_single : M=128, N=256, K=512, A and B ~ N(0,1)                       (seed 1)
  decode_sweep : M in {64,128} x six (N,K); A rows scaled by 10**U(-2,2)       (seeds 2000+i)
  prefill      : M=4096 x the same six (N,K)                                   (seeds 3000+i)
  contiguous   : (G, M per group) in {(4,8192),(8,4096)} x (N,K) in {(4096,7168),(7168,2048)}
                                                                              (seeds 4000+i)
  masked       : (G, Mmax) in {(1,1024),(2,512),(4,256)} x the same two (N,K);
                 masked_m: group 0 empty and group G-1 full for G >= 2, others
                 uniform in [0, Mmax] (stream s+100); G = 1 uses Mmax        (seeds 5000+i)
"""
from __future__ import annotations

NK_PAIRS = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]
GROUPED_NK = [(4096, 7168), (7168, 2048)]


def dense_single():
    return [dict(name="dense_128x256x512", seed=1, M=128, N=256, K=512, row_scaled=False)]


def decode_sweep():
    out = []
    i = 0
    for M in (64, 128):
        for N, K in NK_PAIRS:
            out.append(dict(name=f"decode_M{M}_N{N}_K{K}", seed=2000 + i, M=M, N=N, K=K, row_scaled=True))
            i += 1
    return out


def prefill():
    return [dict(name=f"prefill_M4096_N{N}_K{K}", seed=3000 + i, M=4096, N=N, K=K, row_scaled=False)
            for i, (N, K) in enumerate(NK_PAIRS)]


def contiguous():
    out = []
    i = 0
    for G, Mg in ((4, 8192), (8, 4096)):
        for N, K in GROUPED_NK:
            out.append(dict(name=f"contig_G{G}_M{Mg}_N{N}_K{K}", seed=4000 + i, G=G, M_per_group=Mg, N=N, K=K))
            i += 1
    return out


def masked():
    out = []
    i = 0
    for G, Mmax in ((1, 1024), (2, 512), (4, 256)):
        for N, K in GROUPED_NK:
            out.append(dict(name=f"masked_G{G}_Mmax{Mmax}_N{N}_K{K}", seed=5000 + i, G=G, Mmax=Mmax, N=N, K=K))
            i += 1
    return out
