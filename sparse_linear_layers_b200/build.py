"""Build the Sparse-BitLinear shared library (libsbl.so) in-tree for sm_100a.

    python -m sparse_linear_layers_b200.build        # or build_library() from Python

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it needs nothing but the driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsbl.so")
SOURCES = ("sbl_api.cu", "prep.cu", "quant.cu", "decode.cu", "decode_mma.cu", "prefill.cu", "prefill_pair.cu", "prefill_sp.cu", "mask_monitor.cu", "backward.cu", "backward_tc.cu", "noalloc.cu", "xq_layout.cu")
ARCH = ("-gencode", "arch=compute_100a,code=sm_100a")


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "sbl.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build_library(force: bool = False, verbose: bool = False, extra=(), lib_path: str = LIB,
                  build_dir: str = "_build") -> str:
    """Compile every kernel into ``libsbl.so`` next to this file; returns its path."""
    if not force and lib_path == LIB and not _stale():
        return lib_path
    out_dir = os.path.join(ROOT, build_dir)
    os.makedirs(out_dir, exist_ok=True)
    nvcc = _nvcc()
    common = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
              "--expt-relaxed-constexpr", *extra]
    objs = []
    for src in SOURCES:
        obj = os.path.join(out_dir, src.replace(".cu", ".o"))
        cmd = [nvcc, *common, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib_path + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True,
                        extra=("-Xptxas", "-v") if "--ptxas" in sys.argv else ()))
