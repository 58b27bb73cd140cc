"""Builds libgqa.so in-tree with nvcc for sm_100a (no torch in the link)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgqa.so")
# the same library with the device-side index checks compiled in (-DGQA_DEBUG)
LIB_DEBUG = os.path.join(PKG, "libgqa_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Compiles libgqa.so (or, with debug=True, libgqa_debug.so) unless it is
    newer than every source."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc, *NVCC_FLAGS, *(["-DGQA_DEBUG"] if debug else []), *extra, "-I", INCLUDE, "-I", CSRC,
           "-shared", "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> None:
    """Both libraries, compiled side by side."""
    import threading
    errs = []

    def one(debug):
        try:
            build(force=force, verbose=verbose, debug=debug)
        except Exception as e:  # noqa: BLE001 -- re-raised below
            errs.append(e)

    ts = [threading.Thread(target=one, args=(d,)) for d in (False, True)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]


if __name__ == "__main__":
    if "--debug" in sys.argv:
        build(force="--force" in sys.argv, verbose=True, debug=True)
    else:
        build(force="--force" in sys.argv, verbose=True,
              extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
