"""Builds the CUDA library libq4.so in-tree for sm_100a (nvcc; no JIT cache).

    python -m weight_only_bit_gemv_b200.build [--force] [--verbose] [--debug]

--verbose passes -Xptxas -v (registers, spills, shared memory per kernel).
--debug builds libq4_debug.so instead: the same sources with -DQ4_DEBUG, in
which every kernel checks the index range of each global load and store
before it is made; a failed check skips the access and sets a bit that
q4_bounds_flags() returns.  The binding loads it when Q4_LIBRARY=debug.
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
LIBRARY = os.path.join(PKG, "libq4.so")
DEBUG_LIBRARY = os.path.join(PKG, "libq4_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale(target: str = LIBRARY) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    target = DEBUG_LIBRARY if debug else LIBRARY
    if not (force or stale(target)):
        return target
    tmp = target + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if debug:
        cmd += ["-DQ4_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += sources() + ["-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(target)}")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
