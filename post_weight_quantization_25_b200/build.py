"""Build libgptq_b200.so in place with nvcc for sm_100a.

Usage: python -m post_weight_quantization_25_b200.build [--force] [--debug]
(or build() from Python).  --debug builds libgptq_b200_debug.so instead: the
same sources with device-side index checks (-DGPTQ_DEVICE_CHECKS, read back
by gptq_device_checks).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgptq_b200.so")
DEBUG_LIB = os.path.join(PKG, "libgptq_b200_debug.so")
SOURCES = ["gptq_api.cu", "hessian_syrk.cu", "cholesky.cu", "sweep.cu", "pack.cu", "hadamard.cu"]
HEADERS = ["gptq_internal.cuh", "sm100_ptx.cuh", "panel_gemm.cuh", "persist.cuh", "stage.cuh", "chol_diag.cuh",
           "fdiv.cuh"]
ROOT = os.path.dirname(PKG)


def _nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "gptq.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _flags(verbose: bool) -> list[str]:
    f = ["-O3", "-lineinfo", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]
    return (["-Xptxas=-v"] + f) if verbose else f


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every source to an object file in parallel (the files share
    no device symbols), then link the shared library (the checked one with
    debug=True)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    from concurrent.futures import ThreadPoolExecutor
    objdir = os.path.join(PKG, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, os.path.splitext(f)[0] + ".o") for f in SOURCES]

    def compile_one(i: int) -> None:
        cmd = [_nvcc()] + _flags(verbose) + (["-DGPTQ_DEVICE_CHECKS"] if debug else []) + \
            ["-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
        list(ex.map(compile_one, range(len(SOURCES))))
    cmd = [_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o",
           lib + ".tmp"] + objs
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
