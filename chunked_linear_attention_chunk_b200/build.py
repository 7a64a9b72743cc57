"""Build libkda.so in-tree with nvcc for sm_100a (B200).

    python -m chunked_linear_attention_chunk_b200.build [--verbose-ptxas] [--debug-checks]

The shared library lands next to this file and is what the Python binding loads.  With
--debug-checks (or build(debug_checks=True)) the same sources are built with
KDA_DEBUG_CHECKS into libkda_debug.so, which the binding loads when KDA_DEBUG_CHECKS=1.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkda.so")
LIB_DEBUG = os.path.join(HERE, "libkda_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, debug_checks: bool = False) -> str:
    """Compile every CUDA source into libkda.so, or libkda_debug.so with the kernels' index
    checks (skipped when up to date)."""
    lib = LIB_DEBUG if debug_checks else LIB
    if not force and not ptxas_verbose and not _stale(lib):
        return lib
    cmd = [NVCC, *NVCC_FLAGS]
    if debug_checks:
        cmd += ["-DKDA_DEBUG_CHECKS"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", lib + ".tmp", *sources()]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, debug_checks="--debug-checks" in sys.argv))
