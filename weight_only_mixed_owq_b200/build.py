"""Build the CUDA library libowq_b200.so in-tree with nvcc (sm_100a only).

Usage: python -m weight_only_mixed_owq_b200.build [--force] [--verbose] [--debug-bounds]

--debug-bounds builds libowq_b200_bounds.so instead: the same sources with -DOWQ_DEBUG_BOUNDS
(device index checks that report OWQ_ERR_BOUNDS instead of faulting); load it with
OWQ_LIB_VARIANT=bounds.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libowq_b200.so")
LIB_BOUNDS = os.path.join(PKG, "libowq_b200_bounds.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
         "--expt-relaxed-constexpr", "-cudart", "static"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile every .cu under csrc/ into libowq_b200.so, or with debug_bounds into
    libowq_b200_bounds.so (skipped when up to date)."""
    lib = LIB_BOUNDS if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    extra = ["-DOWQ_DEBUG_BOUNDS"] if debug_bounds else []
    cmd = [nvcc_path(), *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-o", lib + ".tmp", *sources()]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    log = proc.stdout + proc.stderr
    with open(os.path.join(PKG, "build_bounds.log" if debug_bounds else "build.log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if proc.returncode != 0:
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed (see weight_only_mixed_owq_b200/build*.log)")
    os.replace(lib + ".tmp", lib)
    if verbose:
        sys.stdout.write(log)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug_bounds=a.debug_bounds))
