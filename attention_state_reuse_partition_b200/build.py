"""Builds the in-tree CUDA libraries for sm_100a with nvcc: ``libasp.so``
and the checked build ``libasp_debug.so`` (ASP_DEBUG=1: device-side index
checks that report through as_device_status).

Usage: ``python -m attention_state_reuse_partition_b200.build [--verbose]``.
The libraries land next to this file so that they travel with the source
tree.
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
LIB = os.path.join(PKG, "libasp.so")
LIB_DEBUG = os.path.join(PKG, "libasp_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fPIC,-O2", "-shared"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libasp.so")
    return exe


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return all(os.path.getmtime(p) <= t for p in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    """Builds libasp.so, or with debug=True the checked libasp_debug.so."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC]
    if debug:
        cmd += ["-DASP_DEBUG=1"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += sources() + ["-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def build_all(verbose: bool = False, force: bool = False) -> None:
    build(verbose, force)
    build(verbose, force, debug=True)


if __name__ == "__main__":
    build_all(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
    print(LIB_DEBUG)
