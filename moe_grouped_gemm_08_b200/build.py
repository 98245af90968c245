"""Build the sm_100a CUDA library in-tree (nvcc, no JIT): libfp8gemm.so next to this file."""
from __future__ import annotations

import os
import pathlib
import subprocess

HERE = pathlib.Path(__file__).resolve().parent
ROOT = HERE.parent
SO = HERE / "libfp8gemm.so"
SO_DEBUG = HERE / "libfp8gemm_debug.so"  # the same library with the device-side checks (-DFG_DEBUG)
SOURCES = [HERE / "csrc" / "fp8gemm_api.cu"]
DEPENDS = SOURCES + [HERE / "csrc" / "fp8_gemm_kernels.cuh", HERE / "csrc" / "fp8_cast_kernels.cuh",
                     HERE / "csrc" / "sm100_ptx.cuh",
                     ROOT / "include" / "fp8gemm.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(so: pathlib.Path, extra, force: bool, verbose: bool) -> pathlib.Path:
    if not force and so.exists():
        newest = max(p.stat().st_mtime for p in DEPENDS)
        if so.stat().st_mtime >= newest:
            return so
    tmp = so.with_suffix(".so.tmp%d" % os.getpid())
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", str(ROOT / "include"), "-I", str(HERE / "csrc"),
           *(str(s) for s in SOURCES), "-o", str(tmp)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, so)
    return so


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> pathlib.Path:
    """Compile the library (and, with debug=True, its debug build) if any source is newer than
    the built .so."""
    if debug:
        _build_one(SO_DEBUG, ["-DFG_DEBUG"], force, False)
    return _build_one(SO, [], force, verbose)


if __name__ == "__main__":
    print(build(force=True, verbose=True))
