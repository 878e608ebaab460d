"""Build libosdn.so in-tree with nvcc for sm_100a.

Usage: ``python -m delta_rule_recurrent_osdn_b200.build [--verbose-ptxas] [--debug-bounds]``.  The
library is written next to this file; the Python binding loads it from there.  ``--debug-bounds``
writes libosdn_debug.so instead, built with -DOSDN_DEBUG_BOUNDS: the kernels' computed global
stores check their indices and record OSDN_ERR_DEVICE_BOUNDS instead of writing out of bounds
(load it with OSDN_LIBRARY=<path>).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libosdn.so")
DEBUG_LIB = os.path.join(PKG, "libosdn_debug.so")
SOURCES = ["osdn_lib.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libosdn")
    return path


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "osdn.h"))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True,
          debug_bounds: bool = False) -> str:
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    objs = []
    build_dir = os.path.join(PKG, "_build_debug" if debug_bounds else "_build")
    os.makedirs(build_dir, exist_ok=True)
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
               "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
               "--expt-relaxed-constexpr", "-c", os.path.join(CSRC, src), "-o", obj]
        if debug_bounds:
            cmd += ["-DOSDN_DEBUG_BOUNDS"]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {src}")
        if ptxas_verbose or not quiet:
            sys.stderr.write(r.stderr)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, quiet=False,
                debug_bounds=a.debug_bounds))
