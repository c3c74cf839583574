"""Build libsq.so (the sm_100a CUDA kernels + the C ABI of include/sq.h) in-tree."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsq.so")
# the same library with the device-side index checks on (-DSQ_DEBUG_CHECKS): every checked store
# tests its index against its buffer, skips it when outside and reports SQ_ERR_INDEX
LIB_DEBUG = os.path.join(PKG, "libsq_debug.so")
SOURCES = ["sq_api.cu", "sq_quant.cu", "sq_gemm.cu", "sq_svd.cu"]
HEADERS = ["sq_device.cuh", "sq_ptx.cuh", "sq_kernels.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sq.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          debug_checks: bool = False) -> str:
    lib = LIB_DEBUG if debug_checks else LIB
    if not force and not _stale(lib):
        return lib
    if debug_checks:
        extra = list(extra or []) + ["-DSQ_DEBUG_CHECKS"]
    objs = []
    for src in SOURCES:
        obj = os.path.join(CSRC, src.replace(".cu", ".debug.o" if debug_checks else ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs,
                    "-cudart", "static"], check=True)
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None,
          debug_checks="--debug-checks" in sys.argv)
