"""Build the sm_100a shared library ``libcausalconv.so`` in-tree with nvcc.

Usage: ``python -m spectral_sequence_mixing_b200.build`` (also run by
``__graft_entry__.build()``).  nvcc cross-compiles without a GPU.
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
LIB = os.path.join(PKG, "libcausalconv.so")
SOURCES = [os.path.join(CSRC, "api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
# rate probes for the benchmark's --probe mode (not part of the C-ABI library)
PROBE_LIB = os.path.join(PKG, "libccprobe.so")
PROBE_SOURCES = [os.path.join(CSRC, "probe.cu")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_rebuild(lib: str = LIB, deps=DEPS) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps)


def _nvcc(lib: str, sources, verbose: bool, extra_flags) -> None:
    cmd = [nvcc_path(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC, "-shared",
           "-o", lib + ".tmp", *sources]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    if force or needs_rebuild(PROBE_LIB, PROBE_SOURCES):
        _nvcc(PROBE_LIB, PROBE_SOURCES, verbose, extra_flags)
    if force or needs_rebuild():
        _nvcc(LIB, SOURCES, verbose, extra_flags)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None)
