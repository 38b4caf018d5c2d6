"""Builds librglru.so (the CUDA library behind include/rglru.h) in-tree with nvcc.

    python -m lm_causal_depthwise_b200.build          # build if sources changed
    python -m lm_causal_depthwise_b200.build --force  # rebuild

Target: sm_100a only (B200).  The CUDA runtime is linked statically, so the
library does not depend on which libcudart the host process has loaded.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "librglru.so")
BUILD_DIR = os.path.join(PKG, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


TRACE_LIB = os.path.join(PKG, "librglru_trace.so")


def build(force: bool = False, verbose: bool = False, extra_flags=(), out: str = LIB) -> str:
    """Compile every csrc/*.cu for sm_100a and link ``out``.  ``build_trace()``
    makes the per-role timeline variant (-DRGLRU_TRACE) used for kernel studies."""
    if not force and up_to_date() and out == LIB:
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    tag = "" if out == LIB else os.path.splitext(os.path.basename(out))[0] + "."
    for src in sources():
        obj = os.path.join(BUILD_DIR, tag + os.path.basename(src) + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-Xcompiler", "-fPIC"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_trace(verbose: bool = False) -> str:
    return build(force=True, verbose=verbose, extra_flags=("-DRGLRU_TRACE",), out=TRACE_LIB)


if __name__ == "__main__":
    if "--trace" in sys.argv:
        print(build_trace(verbose=True))
    else:
        build(force="--force" in sys.argv, verbose=True)
        print(LIB)
