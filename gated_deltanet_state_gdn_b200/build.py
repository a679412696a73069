"""Build libgdn.so in-tree with nvcc for sm_100a.

    python -m gated_deltanet_state_gdn_b200.build [--force] [--checked | --all]

The library links the CUDA runtime statically and needs no libcuda at link
time (the driver entry points it uses are fetched at run time), so it loads on
a machine without a GPU for the symbol checks.

--checked builds libgdn_checked.so instead: the same sources compiled with
GDN_CHECKS, where every global access and every data-dependent shared-memory
access is tested against its buffer first (an access outside it is skipped and
GDN_DEV_BOUNDS set in the status word).  It is a test build, slower than the
product library; --all builds both.
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
LIB = os.path.join(PKG, "libgdn.so")
LIB_CHECKED = os.path.join(PKG, "libgdn_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    out = LIB_CHECKED if checked else LIB
    if not force and not _stale(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + f".tmp{os.getpid()}"
    defs = ["-DGDN_CHECKS"] if checked else []
    cmd = [nvcc, *NVCC_FLAGS, *defs, *extra, "-I", INCLUDE, "-I", CSRC, "-shared", "-o", tmp,
           *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_all(force: bool = False, verbose: bool = False) -> list:
    """The product library and the checked test build."""
    return [build(force, verbose), build(force, verbose, checked=True)]


if __name__ == "__main__":
    force = "--force" in sys.argv
    if "--all" in sys.argv:
        print(build_all(force, verbose=True))
    else:
        print(build(force, verbose=True, checked="--checked" in sys.argv))
