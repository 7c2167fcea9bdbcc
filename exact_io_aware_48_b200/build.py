"""Build libfa.so (the C-ABI attention library) in-tree with nvcc for sm_100a.

Usage: python -m exact_io_aware_48_b200.build [--force] [--no-debug]

Also builds libfa_debug.so, the same library compiled with FA_DEBUG=1 (device-side index checks; see fa.h).
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
LIB = os.path.join(PKG, "libfa.so")
DEBUG_LIB = os.path.join(PKG, "libfa_debug.so")  # FA_DEBUG=1: device-side index checks (see fa.h)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "fa.h")])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def _compile(lib: str, extra: list, log: str):
    """Start nvcc for one library variant; returns (process, temporary output path, ptxas log path)."""
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "fa_lib.cu"),
           os.path.join(CSRC, "fa_noalloc.cu")]
    return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True), tmp, log


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build libfa.so and (debug=True) libfa_debug.so, the FA_DEBUG=1 variant, in parallel.  Returns LIB."""
    jobs = []
    if force or not up_to_date(LIB):
        jobs.append((LIB, _compile(LIB, [], os.path.join(PKG, "build_ptxas.log"))))
    if debug and (force or not up_to_date(DEBUG_LIB)):
        jobs.append((DEBUG_LIB, _compile(DEBUG_LIB, ["-DFA_DEBUG=1"], os.path.join(PKG, "build_ptxas_debug.log"))))
    for lib, (proc, tmp, log) in jobs:
        _, err = proc.communicate()
        if proc.returncode != 0:
            raise RuntimeError(f"nvcc failed for {os.path.basename(lib)} ({proc.returncode}):\n{err[-6000:]}")
        with open(log, "w") as f:
            f.write(err)
        if verbose:
            sys.stderr.write(err)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--no-debug" not in sys.argv))
