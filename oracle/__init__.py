"""CPU oracle for the FP8 (e4m3) block-scaled NT GEMM -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The CUDA library never does, and this package never
imports the CUDA library: the two share no code.

The arithmetic lives in ``fp8gemm_oracle.c`` (plain C11, fp64, OpenMP over rows,
built with -ffp-contract=off); this module only marshals numpy arrays.

Definition (per output element, scale granularities 1x128 for A and 128x128
for B):
    S_kb   = sum over the 128-wide K block kb of dec(A[m,k]) * dec(B[n,k])
    C[m,n] = bf16_rne( sum_kb S_kb * sfa[kb, m] * sfb[n // 128, kb] )
Sources: the "DeepGEMM" how-to (aisharenet.com), "Main functions" 1-3 (the three
entry points, FP8 in, BF16 out); the turtlesai.it summary (NT layout only,
fine-grained scaling, two-level accumulation); the senqingzn.com news article,
optimisation paragraph (promotion of the FP8 tensor-core partial sums).
Every function here is pinned by the CPU tests in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
_SO = _HERE / "liboracle.so"
_LIB = None


def build(force: bool = False) -> pathlib.Path:
    """Compile the oracle with gcc (plain C11, no fused multiply-add, OpenMP)."""
    src = _HERE / "fp8gemm_oracle.c"
    if force or not _SO.exists() or _SO.stat().st_mtime < src.stat().st_mtime:
        tmp = _SO.with_suffix(".so.tmp%d" % os.getpid())
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", str(src), "-o", str(tmp), "-lm"])
        os.replace(tmp, _SO)
    return _SO


def load(path) -> ctypes.CDLL:
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(str(path))
    vp, c_int, c_long = ctypes.c_void_p, ctypes.c_int, ctypes.c_long
    lib.oracle_e4m3_decode_table.argtypes = [vp]
    lib.oracle_bf16_from_f64.restype = ctypes.c_uint16
    lib.oracle_bf16_from_f64.argtypes = [ctypes.c_double]
    lib.oracle_e5m2_decode_table.argtypes = [vp]
    lib.oracle_gemm_nt.argtypes = [vp, vp, c_long, vp, vp, c_int, c_int, c_int, vp, vp, c_int, c_int]
    lib.oracle_gemm_nt_rows.argtypes = [vp, vp, c_long, vp, vp, c_int, c_int, c_int,
                                        vp, c_int, vp, vp, c_int, c_int]
    lib.oracle_grouped_contiguous.argtypes = [vp, vp, c_long, vp, vp, vp, c_int, c_int,
                                              c_int, c_int, vp, c_int, vp, vp, c_int, c_int]
    lib.oracle_grouped_masked.argtypes = [vp, vp, c_long, vp, vp, vp, c_int, c_int,
                                          c_int, c_int, vp, vp, c_int, c_int]
    lib.oracle_num_threads.restype = c_int
    lib.oracle_e4m3_encode_array.argtypes = [vp, c_long, vp]
    lib.oracle_e5m2_encode_array.argtypes = [vp, c_long, vp]
    lib.oracle_quantize_rows.argtypes = [vp, c_int, c_int, c_int, vp, vp, c_long, c_int]
    lib.oracle_quantize_blocks.argtypes = [vp, c_int, c_int, c_int, vp, vp, c_int]
    return lib


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = load(build())
    return _LIB


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def e4m3_decode_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _lib().oracle_e4m3_decode_table(_p(out))
    return out


def e5m2_decode_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _lib().oracle_e5m2_decode_table(_p(out))
    return out


def bf16_from_f64(x: float) -> int:
    return int(_lib().oracle_bf16_from_f64(float(x)))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


FORMATS = {"e4m3": 0, "e5m2": 1}


def _fmt(f) -> int:
    return FORMATS[f] if isinstance(f, str) else int(f)


def gemm_nt(A, sfa, B, sfb, want_acc: bool = False, rows=None, fmt_a="e4m3", fmt_b="e4m3"):
    """Dense C = A . B^T.  A[M,K] fp8 codes (fmt_a: e4m3 or e5m2), sfa[KB, ld], B[N,K] (fmt_b),
    sfb[NB, KB].

    Returns bf16 bit patterns (uint16 [M or len(rows), N]) and, if asked, the fp64
    values before the final rounding.
    """
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    M, K = A.shape
    N = B.shape[0]
    ld = sfa.shape[1]
    nrows = M if rows is None else len(rows)
    C = np.zeros((nrows, N), dtype=np.uint16)
    acc = np.zeros((nrows, N), dtype=np.float64) if want_acc else None
    if rows is None:
        _lib().oracle_gemm_nt(_p(A), _p(sfa), ld, _p(B), _p(sfb), M, N, K, _p(C), _p(acc),
                              _fmt(fmt_a), _fmt(fmt_b))
    else:
        r = _c(rows, np.int32)
        assert r.size == 0 or (r.min() >= 0 and r.max() < M)
        _lib().oracle_gemm_nt_rows(_p(A), _p(sfa), ld, _p(B), _p(sfb), M, N, K,
                                   _p(r), int(r.size), _p(C), _p(acc), _fmt(fmt_a), _fmt(fmt_b))
    return (C, acc) if want_acc else C


def grouped_contiguous(A, sfa, B, sfb, m_indices, C=None, rows=None, want_acc: bool = False,
                       fmt_a="e4m3", fmt_b="e4m3"):
    """M-grouped contiguous: A[M_total,K], B[G,N,K], sfb[G,NB,KB], m_indices[M_total].

    Rows with m_indices == -1 are left as they are in ``C`` (zeros if C is None).
    With ``rows``, computes only those rows, into a [len(rows), N] array.
    """
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    mi = _c(m_indices, np.int32)
    M_total, K = A.shape
    G, N = B.shape[0], B.shape[1]
    ld = sfa.shape[1]
    nrows = M_total if rows is None else len(rows)
    if C is None:
        C = np.zeros((nrows, N), dtype=np.uint16)
    else:
        C = np.array(C, dtype=np.uint16, copy=True, order="C")
    acc = np.zeros((nrows, N), dtype=np.float64) if want_acc else None
    r = None if rows is None else _c(rows, np.int32)
    _lib().oracle_grouped_contiguous(_p(A), _p(sfa), ld, _p(B), _p(sfb), _p(mi), M_total, G,
                                     N, K, _p(r), 0 if r is None else int(r.size), _p(C), _p(acc),
                                     _fmt(fmt_a), _fmt(fmt_b))
    return (C, acc) if want_acc else C


def grouped_masked(A, sfa, B, sfb, masked_m, C=None, want_acc: bool = False, fmt_a="e4m3", fmt_b="e4m3"):
    """M-grouped masked: A[G,Mmax,K], sfa[G,KB,ld], B[G,N,K], sfb[G,NB,KB], masked_m[G].

    Rows at or past masked_m[g] keep their values from ``C`` (zeros if C is None).
    """
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.float32), _c(sfb, np.float32)
    mm = _c(masked_m, np.int32)
    G, Mmax, K = A.shape
    N = B.shape[1]
    ld = sfa.shape[2]
    if C is None:
        C = np.zeros((G, Mmax, N), dtype=np.uint16)
    else:
        C = np.array(C, dtype=np.uint16, copy=True, order="C")
    acc = np.zeros((G, Mmax, N), dtype=np.float64) if want_acc else None
    _lib().oracle_grouped_masked(_p(A), _p(sfa), ld, _p(B), _p(sfb), _p(mm), G, Mmax, N, K,
                                 _p(C), _p(acc), _fmt(fmt_a), _fmt(fmt_b))
    return (C, acc) if want_acc else C


# ---------------------------------------------------------------------------- the cast step
def e4m3_encode(v) -> np.ndarray:
    """e4m3 codes (uint8) of finite fp32 values: round to nearest, ties to even, saturating."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _lib().oracle_e4m3_encode_array(_p(v), int(v.size), _p(out))
    return out


def e5m2_encode(v) -> np.ndarray:
    """e5m2 codes (uint8) of finite fp32 values: round to nearest, ties to even, saturating."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _lib().oracle_e5m2_encode_array(_p(v), int(v.size), _p(out))
    return out


def quantize_rows(X_bits, ld=None, fmt="e4m3"):
    """A side of the cast: X_bits bf16 bit patterns [M,K] or [G,M,K] -> (codes of the same shape,
    sfa [KB, ld] or [G, KB, ld]); one fp32 scale per 1x128 block of a row, column-major."""
    X = _c(X_bits, np.uint16)
    squeeze = X.ndim == 2
    if squeeze:
        X = X[None]
    G, M, K = X.shape
    KB = (K + 127) // 128
    ld = ld if ld is not None else (M + 3) // 4 * 4
    Q = np.empty(X.shape, dtype=np.uint8)
    sfa = np.zeros((G, KB, ld), dtype=np.float32)
    _lib().oracle_quantize_rows(_p(X), G, M, K, _p(Q), _p(sfa), ld, _fmt(fmt))
    return (Q[0], sfa[0]) if squeeze else (Q, sfa)


def quantize_blocks(X_bits, fmt="e4m3"):
    """B side of the cast: X_bits bf16 bit patterns [N,K] or [G,N,K] -> (codes, sfb [NB,KB] or
    [G,NB,KB]); one fp32 scale per 128x128 block."""
    X = _c(X_bits, np.uint16)
    squeeze = X.ndim == 2
    if squeeze:
        X = X[None]
    G, N, K = X.shape
    Q = np.empty(X.shape, dtype=np.uint8)
    sfb = np.empty((G, (N + 127) // 128, (K + 127) // 128), dtype=np.float32)
    _lib().oracle_quantize_blocks(_p(X), G, N, K, _p(Q), _p(sfb), _fmt(fmt))
    return (Q[0], sfb[0]) if squeeze else (Q, sfb)
