"""Build the KDA C-ABI shared library for sm_100a with nvcc.

The library is built in-tree (``gated_delta_rule_136_b200/_build``) so it
travels with the source tree.  ``python -m gated_delta_rule_136_b200.build``
builds it; :func:`build` is what the binding calls when the library is
missing or older than its sources.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIB_NAME = "libkda_b200.so"
LIB_PATH = os.path.join(BUILD_DIR, LIB_NAME)
# The debug variant: the same sources with -DKDA_DEBUG, whose kernels check
# each unit's token range, sequence and head on the device and record
# KDA_ERR_DEVICE_BOUNDS instead of touching memory outside them.  The binding
# loads it when the environment sets KDA_DEBUG_LIBRARY=1.
DEBUG_LIB_PATH = os.path.join(BUILD_DIR, "libkda_b200_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the KDA CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug: bool = False) -> str:
    """Compile every ``csrc/*.cu`` into one shared library; returns its path
    (``debug``: the variant with device-side argument checks)."""
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not is_stale(path):
        return path
    os.makedirs(BUILD_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared",
           "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", *(["-DKDA_DEBUG"] if debug else []),
           "-I", INCLUDE, "-I", CSRC, *sources(), "-o", tmp]
    if ptxas_info:
        cmd[1:1] = ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv,
                debug="--debug" in sys.argv))
