"""Builds libmuonb200.so in-tree with nvcc for sm_100a.

    python -m muon_optimizer_step_02_b200._build

The library links the CUDA runtime statically and resolves the one driver
entry point it needs (tensor-map encoding) at run time, so it loads on a
machine without a GPU driver.
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
LIB = os.path.join(PKG, "libmuonb200.so")
# The same sources with MUON_DEVICE_CHECKS: every work item and epilogue
# store checked on the device before the access (tests and debugging).
LIB_CHECKED = os.path.join(PKG, "libmuonb200_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) +
                  glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build libmuonb200.so")


def _compile(lib: str, extra, verbose: bool):
    cu = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    tmp = lib + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *cu]
    if verbose:
        print(" ".join(cmd), flush=True)
    return tmp, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                 text=True)


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds the default library and the device-checked one (in parallel)
    when their sources changed; returns the default library's path."""
    jobs = []
    for lib, extra in ((LIB, []), (LIB_CHECKED, ["-DMUON_DEVICE_CHECKS"])):
        if force or is_stale(lib):
            jobs.append((lib, *_compile(lib, extra, verbose)))
    for lib, tmp, proc in jobs:
        out, err = proc.communicate()
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + out + err)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
