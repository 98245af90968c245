"""Python binding of the B200 FP8 block-scaled NT GEMM library (libfp8gemm.so).

Argument marshalling only: every step of the GEMM runs in the CUDA kernels of the
library.  PyTorch supplies device memory and the current stream.  If the compiled
library is missing, importing this package raises -- there is no fallback path.

Entry points (names after the DeepGEMM how-to, aisharenet.com, "Main functions"):
  gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, C=None)
  m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(A, sfa, B, sfb, m_indices, C=None)
  m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, masked_m, C=None)
  get_m_alignment_for_contiguous_layout(), sfa_ld(M)
Layouts: A [M,K] / [G,Mmax,K] e4m3 (uint8 or float8_e4m3fn); sfa fp32 column-major
per K block, [KB, sfa_ld(M)] / [G, KB, sfa_ld(Mmax)]; B [N,K] / [G,N,K]; sfb fp32
[NB, KB] / [G, NB, KB]; C bf16 [M,N] / [G,Mmax,N].  See include/fp8gemm.h.
"""
from __future__ import annotations

import ctypes
import pathlib

import torch

_HERE = pathlib.Path(__file__).resolve().parent
LIB_PATH = _HERE / "libfp8gemm.so"

if not LIB_PATH.exists():
    raise ImportError(f"{LIB_PATH} is not built; run `python moe_grouped_gemm_08_b200/build.py` "
                      "or __graft_entry__.build()")

_vp, _int = ctypes.c_void_p, ctypes.c_int


def _declare(l: ctypes.CDLL) -> ctypes.CDLL:
    """Argument and result types of every C ABI entry point (include/fp8gemm.h)."""
    l.fg_init.argtypes = [_int]
    l.fg_init.restype = _int
    l.fg_shutdown.argtypes = []
    l.fg_shutdown.restype = None
    l.fg_m_alignment.restype = _int
    l.fg_sfa_ld.argtypes = [_int]
    l.fg_sfa_ld.restype = _int
    l.fp8_gemm_nt.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _vp]
    l.fp8_gemm_nt.restype = _int
    l.fp8_gemm_grouped_contiguous.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _vp]
    l.fp8_gemm_grouped_contiguous.restype = _int
    l.fp8_gemm_grouped_masked.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _vp]
    l.fp8_gemm_grouped_masked.restype = _int
    l.fp8_gemm_nt_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _vp]
    l.fp8_gemm_nt_noalloc.restype = _int
    l.fp8_gemm_nt_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _vp]
    l.fp8_gemm_nt_ex.restype = _int
    l.fp8_gemm_grouped_contiguous_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                                                 _vp]
    l.fp8_gemm_grouped_contiguous_ex.restype = _int
    l.fp8_gemm_grouped_masked_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _vp]
    l.fp8_gemm_grouped_masked_ex.restype = _int
    l.fp8_cast_rows.argtypes = [_vp, _vp, _vp, _int, _int, _int, _vp]
    l.fp8_cast_rows.restype = _int
    l.fp8_cast_blocks.argtypes = [_vp, _vp, _vp, _int, _int, _int, _vp]
    l.fp8_cast_blocks.restype = _int
    l.fp8_cast_rows_ex.argtypes = [_vp, _vp, _vp, _int, _int, _int, _int, _vp]
    l.fp8_cast_rows_ex.restype = _int
    l.fp8_cast_blocks_ex.argtypes = [_vp, _vp, _vp, _int, _int, _int, _int, _vp]
    l.fp8_cast_blocks_ex.restype = _int
    l.fg_noalloc_status.argtypes = [_vp]
    l.fg_noalloc_status.restype = _int
    l.fg_get_device_status.argtypes = [_vp]
    l.fg_get_device_status.restype = _int
    l.fg_status_string.argtypes = [_int]
    l.fg_status_string.restype = ctypes.c_char_p
    l.fg_set_dense_path.argtypes = [_int]
    l.fg_set_dense_path.restype = _int
    l.fg_debug_set_stall.argtypes = [_int]
    l.fg_debug_set_stall.restype = _int
    l.fg_set_tile_order.argtypes = [_int]
    l.fg_set_tile_order.restype = _int
    l.fg_set_jit.argtypes = [_int]
    l.fg_set_jit.restype = _int
    l.fg_jit_cache_size.argtypes = []
    l.fg_jit_cache_size.restype = _int
    l.fg_jit_compile_check.argtypes = [_int, _int, _int, ctypes.POINTER(ctypes.c_size_t)]
    l.fg_jit_compile_check.restype = _int
    l.fg_set_pair_promotion.argtypes = [_int]
    l.fg_set_pair_promotion.restype = _int
    l.fg_tile_plan.argtypes = [_int, _int, _int, _int, _int]
    l.fg_tile_plan.restype = _int
    l.fg_set_tile_n.argtypes = [_int]
    l.fg_set_tile_n.restype = _int
    l.fg_set_tiled_streamk.argtypes = [_int]
    l.fg_set_tiled_streamk.restype = _int
    l.fg_set_stage_kblocks.argtypes = [_int]
    l.fg_set_stage_kblocks.restype = _int
    l.fg_set_swap_schedule.argtypes = [_int]
    l.fg_set_swap_schedule.restype = _int
    l.fg_swap_plan.argtypes = [_int, _int, _int]
    l.fg_swap_plan.restype = _int
    l.fg_workspace_bytes.argtypes = []
    l.fg_workspace_bytes.restype = ctypes.c_size_t
    l.fp8_gemm_nt_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, ctypes.c_uint, _vp,
                                 ctypes.c_size_t, _vp]
    l.fp8_gemm_nt_ws.restype = _int
    l.fp8_gemm_grouped_contiguous_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                                                 ctypes.c_uint, _vp, ctypes.c_size_t, _vp]
    l.fp8_gemm_grouped_contiguous_ws.restype = _int
    l.fp8_gemm_grouped_masked_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                                             ctypes.c_uint, _vp, ctypes.c_size_t, _vp]
    l.fp8_gemm_grouped_masked_ws.restype = _int
    l.fg_launch_count.argtypes = []
    l.fg_launch_count.restype = ctypes.c_uint64
    return l


_lib = _declare(ctypes.CDLL(str(LIB_PATH)))

FG_OK = 0
STATUS_NAMES = {i: _lib.fg_status_string(i).decode() for i in range(8)}
lib = _lib  # the raw C ABI, for callers that marshal pointers themselves
DEBUG_LIB_PATH = _HERE / "libfp8gemm_debug.so"
_debug_lib = None


def debug_library() -> ctypes.CDLL:
    """The debug build of the C ABI (libfp8gemm_debug.so, compiled with -DFG_DEBUG): the same
    entry points, with device-side index checks that report FG_ERR_DEVICE_CHECK through its own
    fg_get_device_status.  It keeps its own state (fg_init, workspace, status word)."""
    global _debug_lib
    if _debug_lib is None:
        if not DEBUG_LIB_PATH.exists():
            raise ImportError(f"{DEBUG_LIB_PATH} is not built; run __graft_entry__.build()")
        _debug_lib = _declare(ctypes.CDLL(str(DEBUG_LIB_PATH)))
    return _debug_lib


class FP8GemmError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def _check(code: int, what: str) -> None:
    if code != FG_OK:
        raise FP8GemmError(code, what)


_initialised: set[int] = set()


def init(device: int | None = None) -> None:
    dev = torch.cuda.current_device() if device is None else int(device)
    if dev not in _initialised:
        _check(_lib.fg_init(dev), "fg_init")
        _initialised.add(dev)


def get_m_alignment_for_contiguous_layout() -> int:
    return int(_lib.fg_m_alignment())


def sfa_ld(m: int) -> int:
    return int(_lib.fg_sfa_ld(int(m)))


def set_dense_path(path: int) -> int:
    """0 automatic, 1 one-CTA tiled kernel (dense), 2 swap-AB stream-K (dense, M <= 128),
    3 CTA-pair kernel (dense and masked). Returns the old value."""
    return int(_lib.fg_set_dense_path(int(path)))


def set_tile_n(bn: int) -> int:
    """Output tile width of the tiled / CTA-pair kernels: 0 automatic, or 128, 192, 256. Returns the
    old value."""
    return int(_lib.fg_set_tile_n(int(bn)))


def set_tile_order(order: int) -> int:
    """Tile walk of the tiled family: 0 automatic, 1 m-block groups (m fastest), 2 n fastest."""
    return int(_lib.fg_set_tile_order(int(order)))


def set_jit(enable: bool) -> int:
    """Runtime specialisation of the one-CTA tiled kernel per shape (NVRTC). Returns the old value."""
    return int(_lib.fg_set_jit(1 if enable else 0))


def jit_cache_size() -> int:
    return int(_lib.fg_jit_cache_size())


def jit_compile_check(bn: int, num_kb: int, N: int) -> int:
    """Compile the specialised dense tiled kernel (no GPU needed); returns the cubin size."""
    n = ctypes.c_size_t(0)
    _check(_lib.fg_jit_compile_check(int(bn), int(num_kb), int(N), ctypes.byref(n)), "fg_jit_compile_check")
    return int(n.value)


def set_pair_promotion(warpgroups: int) -> int:
    """Promotion warpgroups of the 256-wide CTA-pair kernel: 2 or 4. Returns the old value."""
    return int(_lib.fg_set_pair_promotion(int(warpgroups)))


def tile_plan(layout: str, M: int, N: int, K: int, G: int = 1) -> int:
    """kernel * 1000 + tile width a call takes (1xxx one-CTA tiled, 3xxx CTA pair, 2000 swap-AB);
    layout "dense", "contiguous" or "masked"; -1 if not applicable."""
    code = {"dense": 0, "contiguous": 1, "masked": 2}[layout]
    return int(_lib.fg_tile_plan(code, int(M), int(N), int(K), int(G)))


def set_tiled_streamk(overhead: int) -> int:
    """Stream-K tail of the tiled kernel: split the last partial wave when its cost (its units +
    `overhead` K blocks + 2.4 per piece summed) is at most one tile (default 18; 0 whenever the last
    wave is partial; negative never). Returns the old value."""
    return int(_lib.fg_set_tiled_streamk(int(overhead)))


def set_swap_schedule(schedule: int) -> int:
    """Small-M kernel schedule: 0 automatic, -1 never the cluster split, 1 whole tiles, 2/4/8 the
    cluster split with that many CTAs per weight tile wherever possible. Returns the old value."""
    return int(_lib.fg_set_swap_schedule(int(schedule)))


def set_stage_kblocks(kps: int) -> int:
    """K blocks per ring stage of the small-M and CTA-pair kernels: 0 automatic (2 when K % 128 == 0),
    1 or 2. Returns the old value."""
    return int(_lib.fg_set_stage_kblocks(int(kps)))


def swap_plan(M: int, N: int, K: int) -> int:
    """Schedule of the small-M kernel for this dense shape: S (2/4/8) cluster split, 1 whole tiles,
    0 stream-K, -1 not applicable."""
    return int(_lib.fg_swap_plan(int(M), int(N), int(K)))


def workspace_bytes(device: int | None = None) -> int:
    """Bytes of a caller-owned split-K workspace for ``device`` (fg_workspace_bytes)."""
    dev = torch.cuda.current_device() if device is None else int(device)
    with torch.cuda.device(dev):
        init(dev)
        return int(_lib.fg_workspace_bytes())


def new_workspace(device=None) -> torch.Tensor:
    """A zero-filled caller-owned workspace (uint8 CUDA tensor) for the GEMM calls of one stream:
    calls that may run at the same time need different workspaces."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else torch.device(device).index)
    return torch.zeros(workspace_bytes(dev.index), dtype=torch.uint8, device=dev)


def _ws(workspace, device):
    """(pointer, bytes) of a caller-owned workspace, (None, 0) for the library's own."""
    if workspace is None:
        return None, 0
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != device:
        raise ValueError(f"workspace must be a contiguous uint8 tensor on {device}")
    return workspace.data_ptr(), workspace.numel()


def launch_count() -> int:
    return int(_lib.fg_launch_count())


def device_status(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(_lib.fg_get_device_status(ctypes.c_void_p(s.cuda_stream)))


FORMATS = {"e4m3": 0, "e5m2": 1}


def _bytes(t: torch.Tensor, what: str, fmt=None):
    """FP8 operand -> (uint8 view, format code).  float8_e4m3fn / float8_e5m2 tensors carry their
    format; uint8 codes are e4m3 unless ``fmt`` ("e4m3" or "e5m2") says otherwise."""
    code = 0
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    elif t.dtype == torch.float8_e5m2:
        t, code = t.view(torch.uint8), 1
    if t.dtype != torch.uint8:
        raise TypeError(f"{what} must be uint8 codes, float8_e4m3fn or float8_e5m2, got {t.dtype}")
    if fmt is not None:
        code = FORMATS[fmt]
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{what} must be a contiguous CUDA tensor")
    return t, code


def _f32(t: torch.Tensor, what: str) -> torch.Tensor:
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{what} must be a contiguous CUDA float32 tensor")
    return t


def _i32(t: torch.Tensor, what: str) -> torch.Tensor:
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{what} must be a contiguous CUDA int32 tensor")
    return t


def _stream(stream, device=None):
    """The stream to launch on: ``stream``, or the current stream of ``device``; a given stream
    must belong to ``device``."""
    if stream is None:
        s = torch.cuda.current_stream(device)
    else:
        s = stream
        if device is not None and s.device != device:
            raise ValueError(f"stream is on {s.device}, the operands on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _same_device(device, **tensors):
    """Every operand must live on the GPU the launch goes to (a pointer into another GPU's or into
    host memory would be dereferenced by the kernel)."""
    for name, t in tensors.items():
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, A on {device}")


def _out(C, shape, device):
    if C is None:
        return torch.empty(shape, dtype=torch.bfloat16, device=device)
    if C.dtype != torch.bfloat16 or tuple(C.shape) != tuple(shape) or not C.is_contiguous():
        raise ValueError(f"C must be a contiguous bfloat16 tensor of shape {tuple(shape)}")
    if C.device != device:
        raise ValueError(f"C is on {C.device}, the operands on {device}")
    return C


def _cdiv(a, b):
    return (a + b - 1) // b


FLAG_STATIC_B = 1  # FG_FLAG_STATIC_B


def gemm_fp8_fp8_bf16_nt(A, sfa, B, sfb, C=None, stream=None, fmt_a=None, fmt_b=None, workspace=None,
                         static_b=False):
    """Dense C[M,N] = A[M,K] . B[N,K]^T with 1x128 (A) and 128x128 (B) fp32 scales; A and B are
    e4m3 or e5m2 (from their dtype, or fmt_a / fmt_b for uint8 codes).  workspace: a caller-owned
    split-K workspace (new_workspace()), else the library's own.  static_b: the caller promises that
    B and sfb are not written by the kernel launched just before on the stream (FG_FLAG_STATIC_B),
    so weight loading may start before that kernel ends."""
    (A, fa), (B, fb) = _bytes(A, "A", fmt_a), _bytes(B, "B", fmt_b)
    sfa, sfb = _f32(sfa, "sfa"), _f32(sfb, "sfb")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K or tuple(sfa.shape) != (_cdiv(K, 128), sfa_ld(M)) or \
            tuple(sfb.shape) != (_cdiv(N, 128), _cdiv(K, 128)):
        raise ValueError("inconsistent shapes")
    dev = A.device
    _same_device(dev, B=B, sfa=sfa, sfb=sfb)
    C = _out(C, (M, N), dev)
    with torch.cuda.device(dev):
        init(dev.index)
        wp, wb = _ws(workspace, dev)
        _check(_lib.fp8_gemm_nt_ws(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), C.data_ptr(),
                                   M, N, K, fa, fb, FLAG_STATIC_B if static_b else 0, wp, wb,
                                   _stream(stream, dev)), "fp8_gemm_nt")
    return C


def m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(A, sfa, B, sfb, m_indices, C=None, stream=None, fmt_a=None,
                                              fmt_b=None, workspace=None):
    """M-grouped contiguous: A[M_total,K], B[G,N,K], m_indices[M_total] (-1 = padding)."""
    (A, fa), (B, fb) = _bytes(A, "A", fmt_a), _bytes(B, "B", fmt_b)
    sfa, sfb, m_indices = _f32(sfa, "sfa"), _f32(sfb, "sfb"), _i32(m_indices, "m_indices")
    M, K = A.shape
    G, N = B.shape[0], B.shape[1]
    if B.shape[2] != K or m_indices.numel() != M or tuple(sfa.shape) != (_cdiv(K, 128), sfa_ld(M)) or \
            tuple(sfb.shape) != (G, _cdiv(N, 128), _cdiv(K, 128)):
        raise ValueError("inconsistent shapes")
    dev = A.device
    _same_device(dev, B=B, sfa=sfa, sfb=sfb, m_indices=m_indices)
    C = _out(C, (M, N), dev)
    with torch.cuda.device(dev):
        init(dev.index)
        wp, wb = _ws(workspace, dev)
        _check(_lib.fp8_gemm_grouped_contiguous_ws(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(),
                                                   C.data_ptr(), m_indices.data_ptr(), M, G, N, K, fa, fb, 0, wp, wb,
                                                   _stream(stream, dev)), "fp8_gemm_grouped_contiguous")
    return C


def m_grouped_gemm_fp8_fp8_bf16_nt_masked(A, sfa, B, sfb, masked_m, C=None, stream=None, fmt_a=None, fmt_b=None,
                                          workspace=None):
    """M-grouped masked: A[G,Mmax,K], masked_m[G] on the device; rows >= masked_m[g] untouched."""
    (A, fa), (B, fb) = _bytes(A, "A", fmt_a), _bytes(B, "B", fmt_b)
    sfa, sfb, masked_m = _f32(sfa, "sfa"), _f32(sfb, "sfb"), _i32(masked_m, "masked_m")
    G, Mmax, K = A.shape
    N = B.shape[1]
    if B.shape[0] != G or B.shape[2] != K or masked_m.numel() != G or \
            tuple(sfa.shape) != (G, _cdiv(K, 128), sfa_ld(Mmax)) or \
            tuple(sfb.shape) != (G, _cdiv(N, 128), _cdiv(K, 128)):
        raise ValueError("inconsistent shapes")
    dev = A.device
    _same_device(dev, B=B, sfa=sfa, sfb=sfb, masked_m=masked_m)
    C = _out(C, (G, Mmax, N), dev)
    with torch.cuda.device(dev):
        init(dev.index)
        wp, wb = _ws(workspace, dev)
        _check(_lib.fp8_gemm_grouped_masked_ws(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(),
                                               C.data_ptr(), masked_m.data_ptr(), G, Mmax, N, K, fa, fb, 0, wp, wb,
                                               _stream(stream, dev)), "fp8_gemm_grouped_masked")
    return C


# ---------------------------------------------------------------------------- the cast step
def _bf16(t: torch.Tensor, what: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{what} must be a contiguous CUDA bfloat16 tensor")
    return t


def cast_fp8_rows(x, stream=None, fmt="e4m3"):
    """A side of the cast: x bf16 [M, K] or [G, M, K] -> (e4m3 codes as uint8, same shape;
    sfa float32 [ceil(K/128), sfa_ld(M)] or [G, ceil(K/128), sfa_ld(M)]), one scale per 1 x 128
    block of a row, in the column-major layout the GEMM entry points read; fmt "e4m3" or "e5m2"."""
    x = _bf16(x, "x")
    grouped = x.dim() == 3
    G, M, K = (x.shape if grouped else (1,) + tuple(x.shape))
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sfa = torch.zeros((G, _cdiv(K, 128), sfa_ld(M)), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        _check(_lib.fp8_cast_rows_ex(x.data_ptr(), q.data_ptr(), sfa.data_ptr(), G, M, K, FORMATS[fmt],
                                     _stream(stream, x.device)), "fp8_cast_rows")
    return q, (sfa if grouped else sfa[0])


def cast_fp8_blocks(w, stream=None, fmt="e4m3"):
    """B side of the cast: w bf16 [N, K] or [G, N, K] -> (e4m3 codes as uint8, same shape;
    sfb float32 [ceil(N/128), ceil(K/128)] or [G, ...]), one scale per 128 x 128 block."""
    w = _bf16(w, "w")
    grouped = w.dim() == 3
    G, N, K = (w.shape if grouped else (1,) + tuple(w.shape))
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sfb = torch.empty((G, _cdiv(N, 128), _cdiv(K, 128)), dtype=torch.float32, device=w.device)
    with torch.cuda.device(w.device):
        _check(_lib.fp8_cast_blocks_ex(w.data_ptr(), q.data_ptr(), sfb.data_ptr(), G, N, K, FORMATS[fmt],
                                       _stream(stream, w.device)), "fp8_cast_blocks")
    return q, (sfb if grouped else sfb[0])
