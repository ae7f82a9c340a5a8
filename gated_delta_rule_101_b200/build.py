"""Builds libkda.so (the CUDA library) in-tree with nvcc for sm_100a.

Usage: ``python -m gated_delta_rule_101_b200.build`` or ``build()`` from Python.
The library is linked against the static CUDA runtime, so it only needs the
NVIDIA driver at run time.
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
LIB = os.path.join(PKG, "libkda.so")
DEBUG_LIB = os.path.join(PKG, "libkda_debug.so")  # the same sources with KDA_DEBUG defined
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or put the CUDA toolkit on PATH")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          debug: bool = False) -> str:
    """Compile every csrc/*.cu into libkda.so (with ``debug``: libkda_debug.so, built with
    KDA_DEBUG defined); returns the library path."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           *(["-DKDA_DEBUG"] if debug else []),
           f"-I{INCLUDE}", f"-I{CSRC}", *(extra or []), "-o", lib + ".tmp", *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr}")
    if verbose and res.stderr:
        print(res.stderr, file=sys.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> list[str]:
    """Both libraries: libkda.so and its KDA_DEBUG variant, compiled in parallel."""
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(2) as ex:
        jobs = [ex.submit(build, force, verbose, None, d) for d in (False, True)]
        return [j.result() for j in jobs]


if __name__ == "__main__":
    if "--ptxas-v" in sys.argv:
        print(build(force=True, verbose=True, extra=["-Xptxas", "-v"], debug="--debug" in sys.argv))
    else:
        print(build_all(force="--force" in sys.argv, verbose=True))
