"""Seeded synthetic inputs for the FP8 block-scaled NT GEMM.

This module only builds inputs; it holds none of the GEMM's arithmetic.  The
CPU oracle's tests and the CUDA path's tests and benchmark both draw from it.

Recipe (shared by every workload):
  * element (r, k) of an operand is normal number ``offset + r*K + k`` of a
    counter-based stream (splitmix64 finaliser, Box-Muller in fp64, fp32 out);
  * A (the token/activation operand) is quantised per 1x128 block along K,
    its fp32 scales stored column-major: ``sfa[kb, m]`` with leading dimension
    ``sfa_ld(M) = ceil(M/4)*4`` so that each K-block column starts 16-byte aligned;
  * B (the weight operand, N x K, or G x N x K) is quantised per 128x128 block,
    ``sfb[(g,) nb, kb]``;
  * quantisation: scale = amax/448 (fp32), code = e4m3_rne_saturating(x/scale).
Seeds: a workload with seed ``s`` draws A from stream ``2*s`` and B from stream
``2*s + 1``; per-row magnitude factors (decode sweep) come from stream ``2*s``
at counter offset 2**62; masked row counts from stream ``s + 100``.
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
_SO = _HERE / "libsynth.so"
_LIB = None
BLOCK = 128
ROW_FACTOR_OFFSET = 1 << 62


def build(force: bool = False) -> pathlib.Path:
    """Compile synth.c into libsynth.so (gcc, OpenMP)."""
    src = _HERE / "synth.c"
    if force or not _SO.exists() or _SO.stat().st_mtime < src.stat().st_mtime:
        tmp = _SO.with_suffix(".so.tmp%d" % os.getpid())
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fopenmp",
                               "-fPIC", "-shared", str(src), "-o", str(tmp), "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    if _LIB is None:
        build()
        lib = ctypes.CDLL(str(_SO))
        u64, i64, c_int = ctypes.c_uint64, ctypes.c_long, ctypes.c_int
        vp = ctypes.c_void_p
        lib.synth_u64.restype = u64
        lib.synth_u64.argtypes = [u64, u64]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, vp]
        lib.synth_uniform_f64.argtypes = [u64, u64, i64, vp]
        lib.synth_e4m3_encode.restype = ctypes.c_uint8
        lib.synth_e4m3_encode.argtypes = [ctypes.c_float]
        lib.synth_quantize_1x128.argtypes = [vp, i64, c_int, vp, vp, i64]
        lib.synth_quantize_128x128.argtypes = [vp, i64, c_int, vp, vp]
        lib.synth_e5m2_encode.restype = ctypes.c_uint8
        lib.synth_e5m2_encode.argtypes = [ctypes.c_float]
        lib.synth_quantized_matrix.argtypes = [u64, u64, i64, c_int, vp, c_int, vp, vp, i64, c_int]
        _LIB = lib
    return _LIB


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def sfa_ld(m: int) -> int:
    """Leading dimension of the column-major A scales: rows rounded up to 4."""
    return (m + 3) // 4 * 4


def cdiv(a: int, b: int) -> int:
    return (a + b - 1) // b


def normal_f32(stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _lib().synth_normal_f32(stream, offset, n, _ptr(out))
    return out


def uniform_f64(stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _lib().synth_uniform_f64(stream, offset, n, _ptr(out))
    return out


def e4m3_encode(x: float) -> int:
    return int(_lib().synth_e4m3_encode(float(x)))


def quantize_1x128(x: np.ndarray, ld: int | None = None):
    """x[rows, K] fp32 -> (codes uint8 [rows,K], scales fp32 [KB, ld])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, K = x.shape
    ld = sfa_ld(rows) if ld is None else ld
    q = np.empty((rows, K), dtype=np.uint8)
    sf = np.zeros((cdiv(K, BLOCK), ld), dtype=np.float32)
    _lib().synth_quantize_1x128(_ptr(x), rows, K, _ptr(q), _ptr(sf), ld)
    return q, sf


def quantize_128x128(x: np.ndarray):
    """x[rows, K] fp32 -> (codes uint8 [rows,K], scales fp32 [RB, KB])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, K = x.shape
    q = np.empty((rows, K), dtype=np.uint8)
    sf = np.empty((cdiv(rows, BLOCK), cdiv(K, BLOCK)), dtype=np.float32)
    _lib().synth_quantize_128x128(_ptr(x), rows, K, _ptr(q), _ptr(sf))
    return q, sf


FORMATS = {"e4m3": 0, "e5m2": 1}


def e5m2_encode(x: float) -> int:
    return int(_lib().synth_e5m2_encode(float(x)))


def quantized_a(stream: int, rows: int, K: int, ld: int | None = None,
                row_scale: np.ndarray | None = None, offset: int = 0, fmt: str = "e4m3"):
    """Generate and quantise an A operand (1x128 blocks, column-major scales); fmt e4m3 or e5m2
    (scale = amax / 448 or amax / 57344)."""
    ld = sfa_ld(rows) if ld is None else ld
    q = np.empty((rows, K), dtype=np.uint8)
    sf = np.zeros((cdiv(K, BLOCK), ld), dtype=np.float32)
    rs = None if row_scale is None else np.ascontiguousarray(row_scale, dtype=np.float32)
    _lib().synth_quantized_matrix(stream, offset, rows, K, _ptr(rs), 0, _ptr(q), _ptr(sf), ld, FORMATS[fmt])
    return q, sf


def quantized_b(stream: int, rows: int, K: int, offset: int = 0, fmt: str = "e4m3"):
    """Generate and quantise a B operand (128x128 blocks); fmt e4m3 or e5m2."""
    q = np.empty((rows, K), dtype=np.uint8)
    sf = np.empty((cdiv(rows, BLOCK), cdiv(K, BLOCK)), dtype=np.float32)
    _lib().synth_quantized_matrix(stream, offset, rows, K, None, 1, _ptr(q), _ptr(sf), 0, FORMATS[fmt])
    return q, sf


def row_factors(seed: int, rows: int) -> np.ndarray:
    """Per-row magnitudes 10**U(-2, 2) (log-uniform in [1e-2, 1e2]), fp32."""
    u = uniform_f64(2 * seed, ROW_FACTOR_OFFSET, rows)
    return (10.0 ** (4.0 * u - 2.0)).astype(np.float32)


def dense_case(seed: int, M: int, N: int, K: int, row_scaled: bool = False, fmt_a: str = "e4m3",
               fmt_b: str = "e4m3") -> dict:
    """Dense workload: A[M,K], sfa[KB, ld], B[N,K], sfb[NB, KB]; operands in e4m3 or e5m2."""
    rs = row_factors(seed, M) if row_scaled else None
    A, sfa = quantized_a(2 * seed, M, K, row_scale=rs, fmt=fmt_a)
    B, sfb = quantized_b(2 * seed + 1, N, K, fmt=fmt_b)
    return dict(kind="dense", A=A, sfa=sfa, B=B, sfb=sfb, M=M, N=N, K=K, ld=sfa.shape[1], fmt_a=fmt_a,
                fmt_b=fmt_b)


def grouped_b(seed: int, G: int, N: int, K: int, fmt: str = "e4m3"):
    """B[G,N,K] with independent draws per expert; sfb[G, NB, KB]."""
    B = np.empty((G, N, K), dtype=np.uint8)
    sfb = np.empty((G, cdiv(N, BLOCK), cdiv(K, BLOCK)), dtype=np.float32)
    for g in range(G):
        q, sf = quantized_b(2 * seed + 1, N, K, offset=g * N * K, fmt=fmt)
        B[g] = q
        sfb[g] = sf
    return B, sfb


def contiguous_case(seed: int, group_rows, N: int, K: int, align: int = BLOCK, fmt_a: str = "e4m3",
                    fmt_b: str = "e4m3") -> dict:
    """M-grouped contiguous workload.

    group_rows[g] valid rows of expert g; each group is padded up to a multiple of
    ``align`` rows, padding rows carry m_indices = -1 (their A rows are drawn too).
    """
    G = len(group_rows)
    padded = [cdiv(r, align) * align for r in group_rows]
    M_total = int(sum(padded))
    m_indices = np.full(M_total, -1, dtype=np.int32)
    start = 0
    for g, (r, p) in enumerate(zip(group_rows, padded)):
        m_indices[start:start + r] = g
        start += p
    A, sfa = quantized_a(2 * seed, M_total, K, fmt=fmt_a)
    B, sfb = grouped_b(seed, G, N, K, fmt=fmt_b)
    return dict(kind="contiguous", A=A, sfa=sfa, B=B, sfb=sfb, m_indices=m_indices,
                M=M_total, G=G, N=N, K=K, ld=sfa.shape[1], group_rows=list(group_rows))


def masked_counts(seed: int, G: int, Mmax: int) -> np.ndarray:
    """masked_m: for G >= 2, group 0 empty, group G-1 full, the rest uniform in [0, Mmax]."""
    if G == 1:
        return np.array([Mmax], dtype=np.int32)
    u = uniform_f64(seed + 100, 0, G)
    m = np.minimum(np.floor(u * (Mmax + 1)), Mmax).astype(np.int32)
    m[0] = 0
    m[G - 1] = Mmax
    return m


def masked_case(seed: int, G: int, Mmax: int, N: int, K: int, masked_m=None, fmt_a: str = "e4m3",
                fmt_b: str = "e4m3") -> dict:
    """M-grouped masked workload: A[G,Mmax,K], sfa[G,KB,ld], B[G,N,K], sfb[G,NB,KB]."""
    ld = sfa_ld(Mmax)
    KB = cdiv(K, BLOCK)
    A = np.empty((G, Mmax, K), dtype=np.uint8)
    sfa = np.zeros((G, KB, ld), dtype=np.float32)
    for g in range(G):
        q, sf = quantized_a(2 * seed, Mmax, K, ld=ld, offset=g * Mmax * K, fmt=fmt_a)
        A[g] = q
        sfa[g] = sf
    B, sfb = grouped_b(seed, G, N, K, fmt=fmt_b)
    mm = masked_counts(seed, G, Mmax) if masked_m is None else np.asarray(masked_m, dtype=np.int32)
    return dict(kind="masked", A=A, sfa=sfa, B=B, sfb=sfb, masked_m=mm,
                G=G, Mmax=Mmax, N=N, K=K, ld=ld)
